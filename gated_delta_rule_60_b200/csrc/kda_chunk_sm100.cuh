// kda_chunk_sm100.cuh -- fused chunked KDA prefill on B200 tensor cores
// (bf16 inputs, fp32 state, d_k = d_v = 128).
//
// Operator (page "Kimi K3 发布核实与 Moonshot AI 主干架构演变", §3): per head
// the state S (d_k x d_v) is decayed per key channel by a_t, corrected with
// beta_t, k_t, v_t (delta rule) and read by q_t after the update; prefill uses
// a form that is recurrent across chunks and parallel inside a chunk.  Same
// page, "K3 对 Kimi Linear 的进一步修改" bullet 1: log a = -5 sigmoid(g), so the
// cumulative log-decay over a 16-token tile stays in [-80, 0] and reciprocal
// decay scaling fits the BF16 exponent range.
//
// Step algorithm.  The state advances in steps of two 16-token tiles (32
// rows r, start state S0).  Per key channel, b_r is the cumulative log-decay
// from the start of the step and the reference point is m = b_15, the end of
// the first tile, so every scaled exponent lies within one tile's range
// (|b_r - m| <= 80):
//   eps = e^m,  delta = e^{b_31 - m},  gamma = eps * delta (step decay)
//   Kr = K e^{b-m},  Qr = Q e^{b-m},  Kh = K e^{m-b}
//   A_kk = Kr Kh^T,  A_qk = Qr Kh^T   (causal entries are e^{b_r - b_i} <= 1)
//   T = (I + Diag(beta) strict_lower(A_kk))^-1 Diag(beta)     (32 x 32)
//   P = causal(A_qk) T,   Z = Diag(delta) Kh^T T              (d_k x 32)
// (T on the CUDA cores, by 16 x 16 blocks: forward substitution inside the
// diagonal blocks, two small products for the off-diagonal one; every
// product of the step on the tensor cores.)
// With Ke = Kr Diag(eps) = K e^b and Qe = Q e^b the step is exactly
//   W = V - Ke S0,   S_next = Diag(gamma) S0 + Z W,   O = Qe S0 + P W.
// On the tensor cores everything is transposed so that the 128 value
// channels are the MMA M dimension (tensor-memory lanes):
//   MMA1  [(Ke S0)^T | (Qe S0)^T] = bf16(S0)^T [Ke ; Qe]^T       (N = 64, K = 128)
//   MMA2  [O^T | S_next^T] += [V^T | -(Ke S0)^T] [P ; Z]^T      (N = 160, K = 2 x 32)
// (Ke and Qe are Kr and Qr rescaled in place by eps once the A_kk / A_qk
// product has read them.)  The fp32 state lives in tensor memory as the
// accumulator of MMA2: before each step the scan warpgroup replaces it by
// gamma * S0^T (fp32, exact decay) and writes the bf16 operand of MMA1.
// Everything that does not involve S0 (gate, decays, A_kk, A_qk, T, P, Z,
// Ke, Qe) is prepared ahead of time.
//
// CTA = one (sequence, head) chain (a packed batch hands out its chains
// longest first), 512 threads:
//   warps 0-3   scan warpgroup: one thread per value channel; thread 0
//               issues the step products, lane 0 of warp 1 the tile loads,
//               lane 0 of warp 2 the L2 prefetches and the TMA stores of o
//               (full steps go through a shared-memory staging tile).
//   warps 4-15  three prep warpgroups, taking steps in turn: gate and decay,
//               scaled operands (in place in the step's tile slot), the
//               A_kk / A_qk product, forward substitution for T, P, the Z
//               product, and the bf16 operand [P ; Z] of MMA2.
// Inside a warpgroup the stages hand over through named barriers that every
// warp reaches on every step; between warpgroups and with the tensor core,
// through mbarriers.  Every mbarrier wait is bounded; a wait that runs out
// raises the device status word, makes the CTA drain its own copies and
// MMAs, free its tensor memory and return.
//
// What sets the speed.  The scan's chain per step is: MMA1 issue (eight
// tcgen05.mma from one thread), MMA1 round trip, -U, MMA2 issue and round
// trip, the state pass.  The prep warpgroups keep ahead of it, but they
// share every SM sub-partition with a scan warp, so their instruction count
// and, above all, their code size matter: sixteen warps running four roles
// of one large loop contend for the instruction cache.  Hence every wait is
// polled by all lanes (a warp never splits into two issue groups), cold paths
// (partial steps, the final state) are out of line, and the prep's element
// loops are rolled where no register array forces full unrolling.
#pragma once

#include "kda_common.cuh"
#include "sm100_ptx.cuh"
#include "../../include/kda.h"

#include <atomic>
#include <cuda.h>

namespace kda {
namespace prefill {

using namespace kda::sm100;

constexpr int kTile = 16;          // intra-chunk tile
constexpr int kStep = 32;          // tokens per state step (two tiles)
constexpr int kD = 128;            // head size (d_k = d_v)
constexpr int kBatchTok = kStep;   // rows of one TMA box
constexpr int kThreads = 512;
constexpr int kPrep = 3;           // prep warpgroups
constexpr int kSlots = 4;          // steps whose tiles are resident at once

// ---- shared memory map (offsets from a 1024-aligned base) ----
// Tile slot of one step: k, q, g, v as [32 rows][64 ch] 128B-swizzled boxes.
// The gate pass overwrites k, q, g in place with Kr, Qr, Kh; the slot also
// holds [P ; Z], operand B of MMA2 (160 rows x 32 tokens, K-major, no swizzle).
constexpr uint32_t SL_K0 = 0, SL_Q0 = 4096, SL_K1 = 8192, SL_Q1 = 12288;
constexpr uint32_t SL_G0 = 16384, SL_G1 = 20480, SL_V0 = 24576, SL_V1 = 28672;
constexpr uint32_t SL_B2 = 32768;
constexpr uint32_t kSlotBytes = 43008;
// Solve scratch of a prep warpgroup.
// The P product reads 128 rows of its A operand causal(A_qk) (only the first
// 32 are used); the other rows fall on the rest of this scratch region.
constexpr uint32_t kScRow = 144;      // bytes per row of the fp32 scratch matrix (36 floats)
constexpr uint32_t SC_AQ = 0;         // causal(A_qk) bf16, K-major no swizzle: A of the P product
constexpr uint32_t SC_AT = 2048;      // (Diag(beta) strict_lower(A_kk))^T, fp32 [32][36]
constexpr uint32_t SC_TB = 6656;      // T bf16, K-major no swizzle (row = column of T): B of Z and P
constexpr uint32_t kScBytes = 8704;
static_assert(SC_AQ + 128 * 64 <= kScBytes, "P product operand rows");
constexpr uint32_t SM_SLOT = 0;
constexpr uint32_t SM_SC = SM_SLOT + kSlots * kSlotBytes;
constexpr uint32_t SM_GAMMA = SM_SC + kPrep * kScBytes;      // kSlots x 128 fp32
constexpr uint32_t SM_EPS = SM_GAMMA + kSlots * 512;         // kSlots x 128 fp32
constexpr uint32_t SM_DELTA = SM_EPS + kSlots * 512;         // kPrep x 128 fp32
// Output staging for the TMA stores of o: 2 steps x [32 tokens][64 ch] x 2,
// 128B swizzle.
constexpr uint32_t SM_OST = (SM_DELTA + kPrep * 512 + 1023) / 1024 * 1024;
constexpr uint32_t kOstBytes = 8192;
constexpr uint32_t kSmemBytes = SM_OST + 2 * kOstBytes;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;
static_assert(kSlotBytes % 1024 == 0, "slot alignment");

// ---- tensor memory columns ----
constexpr uint32_t COL_UP = 0;       // 32: (Ke S0)^T
constexpr uint32_t COL_O = 32;       // 32: O^T
constexpr uint32_t COL_S = 64;       // 128: S^T accumulator
constexpr uint32_t COL_S16 = 192;    // 64: bf16 S^T, A operand of MMA1
constexpr uint32_t COL_UN = 256;     // 16: bf16 -(Ke S0)^T, A operand of MMA2
constexpr uint32_t COL_PREP = 288;   // kPrep x 64: prep accumulators (A_kk | A_qk, then Z | P)
constexpr uint32_t kTmemCols = 512;
static_assert(COL_PREP + 64 * kPrep <= kTmemCols, "tensor memory map overflow");

// A pipeline stage never waits more than microseconds; give up after ~2 s.
constexpr unsigned long long kWaitLimit = 1ull << 32;

#ifdef KDA_TRACE
// Stage timestamps (clock64) of the chain run by CTA 0; a profiling build only.
enum { TR_SCAN_ISSUE = 0, TR_SCAN_U, TR_SCAN_DONE, TR_SCAN_READY, TR_PREP_FULL, TR_PREP_P1,
       TR_PREP_A, TR_PREP_T, TR_PREP_Z, TR_PREP_B,
       TR_S_M1, TR_S_UST, TR_S_BR, TR_S_LD, TR_S_H0, TR_S_H1, TR_S_OLD, TR_S_FENCE, TR_S_ISSUED,
       TR_EVENTS };
constexpr int kTraceLen = 256;
__device__ unsigned long long g_trace[TR_EVENTS][kTraceLen];
__device__ unsigned long long g_cta_time[1024][3];   // globaltimer start, end, smid
#define KDA_TR(ev, idx)                                                              \
    do {                                                                             \
        if (blockIdx.x == 0 && (idx) < kTraceLen) g_trace[ev][idx] = clock64();     \
    } while (0)
#else
#define KDA_TR(ev, idx) do { } while (0)
#endif

struct Barriers {
    uint64_t slot_full[kSlots];
    uint64_t a_done[kPrep], z_done[kPrep], b_ready[kPrep];
    uint64_t mma1_done, d_done;
    uint64_t drain_scan, drain_prep[kPrep];
    uint64_t never;                  // diagnostic: a barrier nothing arrives on
    float beta_s[kPrep][kStep];
    int stop[kPrep + 1];             // per-warpgroup exit decision (last: scan)
    uint32_t tmem_base;
    int abort_flag;
};

// Launch modes.  kModeChains: one CTA per (sequence, head).  kModeSegLocal
// splits one long sequence per head into G segments (segment 0 of seg0_len
// tokens, the others of seg_len).  The recurrence is linear in (S0, V): from
// a start state S_start a segment ends in M_s S_start + R_s and its outputs
// are o_t = o_t(zero start) + S_start^T (M_{s,t}^T q_t), with M_{s,t} the
// transfer from the segment start to token t.  CTAs [0, H*G) run segment 0
// from the real h0 (final: o and the start state of segment 1) and the later
// segments from zero (R_s, and their zero-start outputs into o); CTAs
// [H*G, H*(2G-1)) run the later segments from the identity with v = 0 (M_s,
// and M_{s,t}^T q_t into a scratch).  seg_combine_kernel then forms the start
// states and the final state, and seg_correct_kernel adds S_start^T times the
// scratch to the outputs of every later segment.
enum { kModeChains = 0, kModeSegLocal = 1 };

struct Params {
    const __nv_bfloat16 *beta;
    const __nv_bfloat16 *z;       // output gate: o * sigmoid(z), or NULL
    const float *h0;
    const int32_t *cu;
    __nv_bfloat16 *o;
    __nv_bfloat16 *om;            // segment modes: outputs of the identity runs, rows from seg0_len
    float *hT;
    int N, H;
    long T_tot;
    int mode, G;
    long seg_len;
    long seg0_len;
    float *ws_R, *ws_M, *ws_S;    // [G][H][128][128] each (segment modes)
    unsigned long long wait_limit;  // bound of a pipeline wait, SM clock cycles
    int stall_step;               // diagnostic: step at which the scan waits on `never` (-1: none)
    int range_step;               // diagnostic: step whose operands CTA 0 records (-1: none)
};

// What one CTA runs: a token range of one head, where its state starts and
// ends, and whether it writes o.
struct Chain {
    int64_t start;
    int L;
    int h;
    bool ok;                 // false: malformed bounds, nothing to do
    const float *h0;         // nullptr = zero start (unless h0_identity)
    bool h0_identity;
    float *hT;               // nullptr = do not write the final state
    bool write_o;
    bool v_zero;             // treat v as zero (transfer-matrix runs)
    bool o_alt;              // write o to the identity-run scratch (Params::om)
    bool gate;               // apply the output gate (gated launches)
};

__device__ __forceinline__ Chain chain_of(const Params &p, int cta) {
    Chain c;
    c.h0_identity = false;
    c.v_zero = false;
    c.write_o = true;
    c.o_alt = false;
    c.gate = true;
    constexpr size_t kSt = (size_t)kD * kD;
    if (p.mode == kModeChains) {
        const int n = cta / p.H;
        c.h = cta % p.H;
        int64_t s0 = 0, s1 = 0;
        c.ok = seq_bounds(p.cu, n, p.N, p.T_tot, s0, s1);
        c.start = s0;
        c.L = c.ok ? (int)(s1 - s0) : 0;
        const size_t unit = (size_t)n * p.H + c.h;
        c.h0 = p.h0 ? p.h0 + unit * kSt : nullptr;
        c.hT = (p.hT && c.ok) ? p.hT + unit * kSt : nullptr;
        return c;
    }
    // One sequence per head, split into segments: its bounds must still be
    // [0, T_tot).  Every CTA checks them before any access; a malformed
    // cu_seqlens is reported and the CTA does nothing.
    int64_t b0 = 0, b1 = 0;
    c.ok = seq_bounds(p.cu, 0, 1, p.T_tot, b0, b1);
    int s;
    if (cta < p.H * p.G) {
        // runs from the real start state (segment 0, final) or from zero (later
        // segments); segment 0 of every head first, so that the longest runs
        // start first
        if (cta < p.H) {
            c.h = cta;
            s = 0;
        } else {
            c.h = (cta - p.H) / (p.G - 1);
            s = 1 + (cta - p.H) % (p.G - 1);
        }
        c.h0 = (s == 0 && p.h0) ? p.h0 + (size_t)c.h * kSt : nullptr;
        c.hT = (s == 0 ? p.ws_S + ((size_t)1 * p.H + c.h) * kSt
                       : p.ws_R + ((size_t)s * p.H + c.h) * kSt);
        c.gate = s == 0;          // later segments are gated after their correction
    } else {
        // runs from the identity with v = 0: the transfer matrix M_s (final
        // state) and M_{s,t}^T q_t (outputs, to the scratch)
        const int i = cta - p.H * p.G;
        c.h = i / (p.G - 1);
        s = 1 + i % (p.G - 1);
        c.h0 = nullptr;
        c.h0_identity = true;
        c.v_zero = true;
        c.o_alt = true;
        c.gate = false;
        c.hT = p.ws_M + ((size_t)s * p.H + c.h) * kSt;
    }
    // segment 0 covers [0, seg0_len); segment s >= 1 starts at
    // seg0_len + (s - 1) seg_len (the last one may be shorter)
    c.start = s == 0 ? 0 : (int64_t)p.seg0_len + (int64_t)(s - 1) * p.seg_len;
    const int64_t rem = p.T_tot - c.start;
    const long len = s == 0 ? p.seg0_len : p.seg_len;
    c.L = (int)(rem < len ? (rem < 0 ? 0 : rem) : len);
    if (!c.ok) {
        c.L = 0;
        c.hT = nullptr;
        c.write_o = false;
    }
    return c;
}

// Chains of a packed batch start longest first: CTA b runs head b % H of the
// sequence whose length ranks b / H in decreasing order (ties by index).
// Blocks are dispatched in index order, so the long chains fill the first
// waves and the tail is made of short ones (longest-processing-time list
// scheduling).  The rank of every sequence is computed by each CTA from the
// lengths in shared memory, which is cheap for the batch sizes below.
constexpr int kOrderMaxSeqs = 512;
static_assert(kOrderMaxSeqs <= kThreads, "one sequence per thread when ranking");

__device__ __forceinline__ int longest_first_cta(const Params &p, int tid) {
    __shared__ int len_s[kOrderMaxSeqs];
    __shared__ int pick;
    if (tid == 0) pick = 0;
    if (tid < p.N) {
        const int64_t d = (int64_t)p.cu[tid + 1] - p.cu[tid];
        len_s[tid] = d < 0 ? -1 : (d > 0x7fffffff ? 0x7fffffff : (int)d);
    }
    __syncthreads();
    // (length descending, index ascending) is a strict total order, so the
    // ranks are a permutation of [0, N) whatever the lengths are, and
    // exactly one thread finds the wanted rank.
    const int want = (int)(blockIdx.x / p.H);
    if (tid < p.N) {
        const int li = len_s[tid];
        int rank = 0;
        for (int j = 0; j < p.N; ++j) {
            const int lj = len_s[j];
            rank += (lj > li) | ((lj == li) & (j < tid));
        }
        if (rank == want) pick = tid;
    }
    __syncthreads();
    return pick * p.H + (int)(blockIdx.x % p.H);
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Warp-uniform bounded wait: every lane polls the barrier and the warp
// agrees on the outcome (a wait counts as completed only if it completed for
// all lanes).  Polling from one lane and broadcasting its result leaves that
// lane in a convergence group of its own after the loop, and the warp then
// issues each later instruction twice, once per group.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity,
                                          volatile int *abort, unsigned long long limit) {
    const bool ok = mbar_wait(bar, parity, abort, limit);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void fail(Barriers &bars) {
    bars.abort_flag = 1;
    raise_error(kErrTimeout);
}

// 32 values of one lane, passed by value to the out-of-line helpers below.
struct OutRegs {
    uint32_t v[kStep];
};

// Diagnostic range record (test-only): magnitudes of one step's scaled
// operands as the kernel forms them.  Rows: Kr, Qr, Kh (bf16, written by the
// gate pass) and Z = Kh^T T (fp32, read from tensor memory before the delta
// rescale).  Columns: max |x| and min nonzero |x| (float bits), then counts of
// subnormals, zeros, non-finite values and all values.
enum { kRangeMax = 0, kRangeMinNz, kRangeSub, kRangeZero, kRangeNonFinite, kRangeCount, kRangeCols };
__device__ unsigned int g_range[4][kRangeCols];

__device__ __forceinline__ void range_add(int row, float m, float mn, unsigned sub, unsigned zero,
                                          unsigned nonfin, unsigned cnt) {
    atomicMax(&g_range[row][kRangeMax], __float_as_uint(m));
    atomicMin(&g_range[row][kRangeMinNz], __float_as_uint(mn));
    atomicAdd(&g_range[row][kRangeSub], sub);
    atomicAdd(&g_range[row][kRangeZero], zero);
    atomicAdd(&g_range[row][kRangeNonFinite], nonfin);
    atomicAdd(&g_range[row][kRangeCount], cnt);
}

// The bf16 operands of the tile slot, after the gate pass (one prep warpgroup).
__device__ __noinline__ void range_probe_operands(const unsigned char *slot, int pt) {
    const uint32_t base[3][2] = {{SL_K0, SL_K1}, {SL_Q0, SL_Q1}, {SL_G0, SL_G1}};
#pragma unroll 1
    for (int row = 0; row < 3; ++row) {
        float m = 0.f, mn = __uint_as_float(0x7f800000u);
        unsigned sub = 0, zero = 0, nonfin = 0, cnt = 0;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            const uint16_t *e = reinterpret_cast<const uint16_t *>(slot + base[row][half]);
#pragma unroll 1
            for (int i = pt; i < kStep * 64; i += 128) {
                const uint16_t b = e[i];
                const uint16_t ex = (b >> 7) & 0xff, man = b & 0x7f;
                const float a = fabsf(__uint_as_float((uint32_t)b << 16));
                ++cnt;
                if (ex == 0xff) { ++nonfin; continue; }
                if (ex == 0 && man == 0) { ++zero; continue; }
                if (ex == 0) ++sub;
                m = fmaxf(m, a);
                mn = fminf(mn, a);
            }
        }
        range_add(row, m, mn, sub, zero, nonfin, cnt);
    }
}

// Z = Kh^T T for this thread's key channel, 32 columns, before the delta rescale.
__device__ __noinline__ void range_probe_z(OutRegs zv) {
    float m = 0.f, mn = __uint_as_float(0x7f800000u);
    unsigned sub = 0, zero = 0, nonfin = 0;
#pragma unroll 1
    for (int c = 0; c < kStep; ++c) {
        const uint32_t b = zv.v[c];
        const uint32_t ex = (b >> 23) & 0xff, man = b & 0x7fffff;
        const float a = fabsf(__uint_as_float(b));
        if (ex == 0xff) { ++nonfin; continue; }
        if (ex == 0 && man == 0) { ++zero; continue; }
        if (ex == 0) ++sub;
        m = fmaxf(m, a);
        mn = fminf(mn, a);
    }
    range_add(3, m, mn, sub, zero, nonfin, kStep);
}

// Diagnostic stall (out of line, off the steady-state instruction stream).
__device__ __noinline__ void stall_here(Barriers &bars, volatile int *abort, unsigned long long limit) {
    if (!warp_wait(&bars.never, 0, abort, limit)) fail(bars);
}

// Barrier among the warps of one warpgroup (id >= 1; 0 is __syncthreads).
__device__ __forceinline__ void group_sync(int id) {
    asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}

// Byte offset of element (row n, k) of a K-major no-swizzle bf16 tile with
// 32 k per row: 8-row x 16-byte core matrices, LBO 128 (next 8 k), SBO 512
// (next 8 rows).
__host__ __device__ __forceinline__ uint32_t core32_off(uint32_t n, uint32_t k) {
    return (n >> 3) * 512u + (k >> 3) * 128u + (n & 7u) * 16u + (k & 7u) * 2u;
}

// Gate, decay and scaled operands of one step, in place in its tile slot.
// Thread (pw, lane) of a prep warpgroup handles rows 16 (pw >> 1) .. + 15
// and key channels 64 (pw & 1) + 2 lane, + 1.  kFull: all 32 rows are tokens
// of the sequence (no masking).  Writes eps (first tile) or delta (second).
// The cumulative log-decay is summed in base 2 (b = sum of -5 log2(e)
// sigmoid(g)), so each element costs two MUFU operations for the sigmoid
// and two for e^{b-m} and its reciprocal.  The first tile's threads sum
// their tile once ahead (m = b_15) so that the main pass is a single loop;
// the loops stay rolled by half, which keeps the prep warps' code small
// enough to share the instruction cache with the scan.
template <bool kFull>
__device__ __forceinline__ void gate_pass(unsigned char *slot, int pw, int lane, int Ls,
                                          float *eps_out, float *dlt_out) {
    const int th = pw >> 1, kb = pw & 1;
    const int r0 = 16 * th;
    const uint32_t oK = kb ? SL_K1 : SL_K0, oQ = kb ? SL_Q1 : SL_Q0;
    const uint32_t oG = kb ? SL_G1 : SL_G0;
    // element (r0 + rr, 2 lane) of a 128-byte-swizzled box: the 16-byte
    // chunk (lane >> 2) of row rr moves to chunk (lane >> 2) ^ (rr & 7)
    const uint32_t cbase = (uint32_t)r0 * 128u + (uint32_t)(lane & 3) * 4u;
    const uint32_t chunk = (uint32_t)(lane >> 2);
    const float2 c1 = make_float2(-kLog2e, -kLog2e);
    const float2 c5 = make_float2(-5.f * kLog2e, -5.f * kLog2e);
    const float2 one = make_float2(1.f, 1.f);
    // first tile: m = b_15, summed first (the same sums as the main loop)
    float2 m = make_float2(0.f, 0.f);
    if (th == 0) {
#pragma unroll 8
        for (int rr = 0; rr < kTile; ++rr) {
            const uint32_t o = cbase + (rr >> 3) * 1024u + (rr & 7) * 128u + ((chunk ^ (rr & 7)) << 4);
            const float2 g = bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(slot + oG + o));
            const float2 x = fmul2(g, c1);
            const float2 den = fadd2(make_float2(ex2(x.x), ex2(x.y)), one);
            const float2 sg = make_float2(rcp(den.x), rcp(den.y));
            if (kFull || r0 + rr < Ls) m = ffma2(sg, c5, m);
        }
    }
    const float2 nbase = make_float2(-m.x, -m.y);
    float2 b = make_float2(0.f, 0.f);
#pragma unroll 8
    for (int rr = 0; rr < kTile; ++rr) {
        const uint32_t o = cbase + (rr >> 3) * 1024u + (rr & 7) * 128u + ((chunk ^ (rr & 7)) << 4);
        const bool live = kFull || r0 + rr < Ls;
        {
            const float2 g = bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(slot + oG + o));
            const float2 x = fmul2(g, c1);
            const float2 den = fadd2(make_float2(ex2(x.x), ex2(x.y)), one);
            const float2 sg = make_float2(rcp(den.x), rcp(den.y));
            if (live) b = ffma2(sg, c5, b);
        }
        const float2 dd = fadd2(b, nbase);
        const float2 er = make_float2(ex2(dd.x), ex2(dd.y));                // e^{b-m}
        const float2 ei = make_float2(rcp(er.x), rcp(er.y));                // e^{m-b}
        const uint32_t kraw = live ? *reinterpret_cast<const uint32_t *>(slot + oK + o) : 0u;
        const uint32_t qraw = live ? *reinterpret_cast<const uint32_t *>(slot + oQ + o) : 0u;
        const float2 kf = bf16x2_to_float2(kraw), qf = bf16x2_to_float2(qraw);
        const float2 kr = fmul2(kf, er), qr = fmul2(qf, er), kh = fmul2(kf, ei);
        *reinterpret_cast<uint32_t *>(slot + oK + o) = pack_bf16(kr.x, kr.y);
        *reinterpret_cast<uint32_t *>(slot + oQ + o) = pack_bf16(qr.x, qr.y);
        *reinterpret_cast<uint32_t *>(slot + oG + o) = pack_bf16(kh.x, kh.y);
    }
    // eps (first tile: b_15 = m) or delta (second tile: b_31 - b_15)
    *reinterpret_cast<float2 *>((th == 0 ? eps_out : dlt_out) + 64 * kb + 2 * lane) =
        make_float2(ex2(b.x), ex2(b.y));
}

// The last, partial step of a sequence: out of line, so that its code stays
// out of the instruction stream of the steady-state loop.
__device__ __noinline__ void gate_pass_partial(unsigned char *slot, int pw, int lane, int Ls,
                                               float *eps_out, float *dlt_out) {
    gate_pass<false>(slot, pw, lane, Ls, eps_out, dlt_out);
}

// Masked plain stores of the last, partial step's outputs (out of line).
__device__ __noinline__ void store_o_partial(__nv_bfloat16 *dst, size_t step, int Lc, OutRegs ov) {
#pragma unroll 1
    for (int r = 0; r < Lc; ++r) dst[(size_t)r * step] = __float2bfloat16_rn(__uint_as_float(ov.v[r]));
}

// One quarter (32 key channels) of the final state of a chain (out of line).
__device__ __noinline__ void store_state_quarter(float *dst, OutRegs sv) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i) dst[(size_t)i * kD] = __uint_as_float(sv.v[i]);
}

// kGate: the fused output gate o * sigmoid(z) (p.z), compiled only into the
// gated instantiation so that the plain operator carries no trace of it.
// kProbe: the diagnostic range record, compiled only into the instantiation
// a kda_debug_range_prefill call launches.
template <bool kGate, bool kProbe = false>
__global__ void __launch_bounds__(kThreads, 1)
chunk_fwd_sm100_kernel(const __grid_constant__ CUtensorMap map_q,
                       const __grid_constant__ CUtensorMap map_k,
                       const __grid_constant__ CUtensorMap map_v,
                       const __grid_constant__ CUtensorMap map_g,
                       const __grid_constant__ CUtensorMap map_o,
                       const __grid_constant__ CUtensorMap map_om,
                       const Params p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzled tiles, as an offset into
    // the shared array, so that every access below stays a shared-memory
    // access with 32-bit addressing
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ Barriers bars;
    volatile int *abortp = &bars.abort_flag;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
#ifdef KDA_TRACE
    if (tid == 0 && blockIdx.x < 1024) {
        unsigned long long t, sid;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        asm volatile("mov.u32 %0, %%smid;" : "=r"(*reinterpret_cast<unsigned *>(&sid)));
        g_cta_time[blockIdx.x][0] = t;
        g_cta_time[blockIdx.x][2] = sid & 0xffffffffu;
    }
#endif
    const bool reorder = p.mode == kModeChains && p.cu != nullptr && p.N > 1 &&
                         p.N <= kOrderMaxSeqs;
    const Chain ch = chain_of(p, reorder ? longest_first_cta(p, tid) : (int)blockIdx.x);
    const int h = ch.h;
    const int64_t start = ch.start;
    const int L = ch.L;
    const int nS = (L + kStep - 1) / kStep;

    if (tid == 0) {
        for (int i = 0; i < kSlots; ++i) mbar_init(&bars.slot_full[i], 1);
        for (int i = 0; i < kPrep; ++i) {
            mbar_init(&bars.a_done[i], 1);
            mbar_init(&bars.z_done[i], 1);
            mbar_init(&bars.b_ready[i], 1);
            mbar_init(&bars.drain_prep[i], 1);
            bars.stop[i] = 0;
        }
        mbar_init(&bars.mma1_done, 1);
        mbar_init(&bars.never, 1);
        mbar_init(&bars.d_done, 1);
        mbar_init(&bars.drain_scan, 1);
        bars.stop[kPrep] = 0;
        bars.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&bars.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncwarp();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = bars.tmem_base;
    const uint32_t s_base = smem_u32(sm);

    if (warp < 4) {
        // ================================================ scan warpgroup
        const int j = tid;                                  // value channel = TMEM lane
        const uint32_t la = (uint32_t)(32 * warp) << 16;
        bool issued = false;
        const float *h0u = ch.h0 ? ch.h0 + j : nullptr;
        constexpr uint32_t id1 = idesc_bf16(128, 64, false, false);
        constexpr uint32_t id2 = idesc_bf16(128, 160, false, false);
        constexpr uint32_t id2v = idesc_bf16(128, 160, true, false);

        int loads = 0;                                      // steps whose tiles were requested
        auto load_step = [&](int s) {     // k, q, g, v rows of step s -> slot s % kSlots
            unsigned char *slot = sm + SM_SLOT + (s % kSlots) * kSlotBytes;
            uint64_t *full = &bars.slot_full[s % kSlots];
            const int z = (int)(start + (int64_t)kStep * s);
            mbar_expect_tx(full, ch.v_zero ? 24576u : 32768u);
            tma_load_3d(slot + SL_K0, &map_k, full, 0, h, z);
            tma_load_3d(slot + SL_K1, &map_k, full, 64, h, z);
            tma_load_3d(slot + SL_Q0, &map_q, full, 0, h, z);
            tma_load_3d(slot + SL_Q1, &map_q, full, 64, h, z);
            tma_load_3d(slot + SL_G0, &map_g, full, 0, h, z);
            tma_load_3d(slot + SL_G1, &map_g, full, 64, h, z);
            if (!ch.v_zero) {
                tma_load_3d(slot + SL_V0, &map_v, full, 0, h, z);
                tma_load_3d(slot + SL_V1, &map_v, full, 64, h, z);
            }
            ++loads;
        };
        auto prefetch_step = [&](int s) {   // warm L2 for a later step
            const int z = (int)(start + (int64_t)kStep * s);
            for (int x = 0; x < 128; x += 64) {
                tma_prefetch_3d(&map_k, x, h, z);
                tma_prefetch_3d(&map_q, x, h, z);
                tma_prefetch_3d(&map_g, x, h, z);
                if (!ch.v_zero) tma_prefetch_3d(&map_v, x, h, z);
            }
        };
        // tile loads come from lane 0 of warp 1 and L2 prefetches from lane 0
        // of warp 2: both are idle while MMA1 runs, off the issuing thread
        const bool loader = tid == 32, prefetcher = tid == 64;
        if (loader && nS > 0) {
            prefetch_tmap(&map_k);
            prefetch_tmap(&map_q);
            prefetch_tmap(&map_g);
            prefetch_tmap(&map_v);
            for (int s = 0; s < kSlots && s < nS; ++s) load_step(s);
        }
        if (prefetcher)
            for (int s = kSlots; s < 2 * kSlots && s < nS; ++s) prefetch_step(s);
        bool alive = nS > 0;
        if (alive) {
            // initial state: gamma_0 * S0 (fp32) and bf16(S0)
            if (warp_wait(&bars.b_ready[0], 0, abortp, p.wait_limit)) {
                const float4 *g4 = reinterpret_cast<const float4 *>(sm + SM_GAMMA);
#pragma unroll 1
                for (int part = 0; part < 4; ++part) {
                    float s0[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int row = 32 * part + i;
                        s0[i] = h0u ? h0u[(size_t)row * kD]
                                    : ((ch.h0_identity && row == j) ? 1.f : 0.f);
                    }
                    uint32_t sb[16], y[32];
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        const float4 gm = g4[8 * part + q4];
                        sb[2 * q4] = pack_bf16(s0[4 * q4], s0[4 * q4 + 1]);
                        sb[2 * q4 + 1] = pack_bf16(s0[4 * q4 + 2], s0[4 * q4 + 3]);
                        y[4 * q4] = __float_as_uint(gm.x * s0[4 * q4]);
                        y[4 * q4 + 1] = __float_as_uint(gm.y * s0[4 * q4 + 1]);
                        y[4 * q4 + 2] = __float_as_uint(gm.z * s0[4 * q4 + 2]);
                        y[4 * q4 + 3] = __float_as_uint(gm.w * s0[4 * q4 + 3]);
                    }
                    tmem_st16(tm + la + COL_S16 + 16 * part, sb);
                    tmem_st16(tm + la + COL_S + 32 * part, *reinterpret_cast<uint32_t(*)[16]>(y));
                    tmem_st16(tm + la + COL_S + 32 * part + 16, *reinterpret_cast<uint32_t(*)[16]>(y + 16));
                }
                tmem_wait_st();
            } else {
                fail(bars);
            }
            tc_fence_before();
            if (tid == 0) bars.stop[kPrep] = *abortp;
            group_sync(1);
            alive = bars.stop[kPrep] == 0;
        } else if (ch.hT) {
            float *dst = ch.hT + j;
            for (int row = 0; row < kD; ++row)
                dst[(size_t)row * kD] = h0u ? h0u[(size_t)row * kD]
                                            : ((ch.h0_identity && row == j) ? 1.f : 0.f);
        }

        // Outputs of a step are held in registers until the next MMA1 has
        // been issued.  A full step goes through shared memory and a TMA
        // store (issued by lane 0 of warp 2 after the next barrier); the last,
        // partial step of a sequence is written with masked plain stores.
        uint32_t ov[32];
        int o_step = -1, o_staged = -1, o_stored = -1;
        const bool o_issuer = tid == 64;
        auto store_o = [&]() {
            if (o_step < 0 || !ch.write_o) { o_step = -1; return; }
            const int Lc = L - kStep * o_step;
            if (kGate && ch.gate) {
                // fused output gate: o * sigmoid(z) on the values in registers
                const __nv_bfloat16 *zr = p.z + ((size_t)(start + kStep * o_step) * p.H + h) * kD + j;
                const size_t step = (size_t)p.H * kD;
#pragma unroll
                for (int r = 0; r < kStep; ++r)
                    if (r < Lc)
                        ov[r] = __float_as_uint(__uint_as_float(ov[r]) *
                                                out_gate(__bfloat162float(zr[(size_t)r * step])));
            }
            if (Lc >= kStep) {
                // lanes j, j ^ 1 swap half of their tokens so that each writes
                // 32-bit words (channels j & ~1, j | 1) of 16 tokens
                unsigned char *st = sm + SM_OST + (o_step & 1) * kOstBytes + (j >> 6) * 4096;
                const bool odd = j & 1;
                const int r_base = odd ? 16 : 0;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint32_t mine = odd ? ov[16 + i] : ov[i];    // token r_base + i, own channel
                    const uint32_t give = odd ? ov[i] : ov[16 + i];    // the partner writes that token
                    const uint32_t got = __shfl_xor_sync(0xffffffffu, give, 1);
                    const float lo = __uint_as_float(odd ? got : mine), hi = __uint_as_float(odd ? mine : got);
                    *reinterpret_cast<uint32_t *>(st + sw128_off(r_base + i, (j & 63) & ~1)) = pack_bf16(lo, hi);
                }
                fence_proxy_async_smem();
                o_staged = o_step;
            } else {
                __nv_bfloat16 *dst =
                    ch.o_alt ? p.om + ((size_t)(start - p.seg0_len + kStep * o_step) * p.H + h) * kD + j
                             : p.o + ((size_t)(start + kStep * o_step) * p.H + h) * kD + j;
                OutRegs orr;
#pragma unroll
                for (int r = 0; r < kStep; ++r) orr.v[r] = ov[r];
                store_o_partial(dst, (size_t)p.H * kD, Lc, orr);
            }
            o_step = -1;
        };
        // after a barrier that follows store_o: write the staged step to global memory
        auto flush_o = [&]() {
            if (!o_issuer || o_staged <= o_stored) return;
            const unsigned char *st = sm + SM_OST + (o_staged & 1) * kOstBytes;
            // the identity runs' scratch holds rows from seg0_len on
            const int z = (int)(start + (int64_t)kStep * o_staged - (ch.o_alt ? p.seg0_len : 0));
            const CUtensorMap *mp = ch.o_alt ? &map_om : &map_o;
            tma_store_3d(mp, st, 0, h, z);
            tma_store_3d(mp, st + 4096, 64, h, z);
            bulk_commit_group();
            o_stored = o_staged;
        };
        for (int c = 0; alive && c < nS; ++c) {
            const int sl = c % kSlots;
            const uint32_t slot_u = s_base + SM_SLOT + sl * kSlotBytes;
            // diagnostic: a wait that nothing completes, so that the bounded
            // wait runs out here and the CTA takes its abort and drain path
            if (c == p.stall_step) stall_here(bars, abortp, p.wait_limit);
            // ---- MMA1: [(Ke S)^T | (Qe S)^T] = bf16(S)^T [Ke ; Qe]^T, then the v part of MMA2
            if (tid == 0 && !*abortp) {
                KDA_TR(TR_SCAN_ISSUE, c);
                tc_fence_after();
                KDA_TR(TR_S_FENCE, c);
                const uint64_t dk = sdesc(slot_u, 16, 1024, kLayoutSW128);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tm + COL_UP, tm + COL_S16 + 8 * kk,
                           sdesc_at(dk, (kk >> 2) * SL_K1 + (kk & 3) * 32), id1, kk > 0);
                tc_commit(&bars.mma1_done);
                KDA_TR(TR_S_ISSUED, c);
                if (!ch.v_zero) {
                    const uint64_t dv = sdesc(slot_u + SL_V0, SL_V1 - SL_V0, 1024, kLayoutSW128);
                    const uint64_t db = sdesc(slot_u + SL_B2, 128, 512, kLayoutNone);
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        mma_ss(tm + COL_O, sdesc_at(dv, 2048 * kk), sdesc_at(db, 256 * kk), id2v, 1);
                }
                issued = true;
            }
            // the slot of step c - 1 was freed by its completed products:
            // request step c - 1 + kSlots (overlaps the MMA1 round trip)
            if (loader && c >= 1 && c - 1 + kSlots < nS && !*abortp) load_step(c - 1 + kSlots);
            if (prefetcher && c >= 1 && c - 1 + 2 * kSlots < nS) prefetch_step(c - 1 + 2 * kSlots);
            // outputs of step c - 1, during the MMA1 round trip (thread 0 after its issue)
            store_o();
            // ---- -(Ke S)^T in bf16: A operand of the second half of MMA2
            if (warp_wait(&bars.mma1_done, c & 1, abortp, p.wait_limit)) {
                if (tid == 0) KDA_TR(TR_S_M1, c);
                tc_fence_after();
                uint32_t u[32], un[16];
                tmem_ld32(tm + la + COL_UP, u);
                tmem_wait_ld();
#pragma unroll
                for (int w = 0; w < 16; ++w)
                    un[w] = pack_bf16(-__uint_as_float(u[2 * w]), -__uint_as_float(u[2 * w + 1]));
                tmem_st16(tm + la + COL_UN, un);
                tmem_wait_st();
                if (tid == 0) KDA_TR(TR_S_UST, c);
            } else {
                fail(bars);
            }
            // staged outputs flushed before this barrier have left shared memory,
            // so the buffer the next store_o writes is free
            if (o_issuer) bulk_wait_group_read<0>();
            tc_fence_before();
            group_sync(1);
            if (!*abortp) flush_o();
            if (tid == 0 && !*abortp) {
                KDA_TR(TR_SCAN_U, c);
                tc_fence_after();
                const uint64_t db = sdesc(slot_u + SL_B2, 128, 512, kLayoutNone);
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                    mma_ts(tm + COL_O, tm + COL_UN + 8 * kk, sdesc_at(db, 256 * kk), id2, 1);
                tc_commit(&bars.d_done);
            }
            // the next step's operands: usually prepared well before MMA2 completes,
            // so this wait runs during the round trip
            const bool has_next = c + 1 < nS;
            bool ready = true;
            if (has_next) ready = warp_wait(&bars.b_ready[(c + 1) % kPrep], ((c + 1) / kPrep) & 1, abortp, p.wait_limit);
            if (!ready) fail(bars);
            // ---- step done: outputs, next step's operands (or the final state)
            if (warp_wait(&bars.d_done, c & 1, abortp, p.wait_limit)) {
                tc_fence_after();
                if (tid == 0) KDA_TR(TR_SCAN_DONE, c);
                if (tid == 0) KDA_TR(TR_S_BR, c);
                const int sn = (c + 1) % kSlots;
                const float4 *g4 = reinterpret_cast<const float4 *>(sm + SM_GAMMA + sn * 512);
                tmem_ld32(tm + la + COL_O, ov);      // waited for with the first quarter
#pragma unroll 1
                for (int qt = 0; qt < 4 && ready; ++qt) {       // 32 key channels at a time
                    uint32_t sv[32];
                    tmem_ld32(tm + la + COL_S + 32 * qt, sv);
                    tmem_wait_ld();
                    if (tid == 0 && qt == 0) KDA_TR(TR_S_LD, c);
                    if (has_next) {
                        uint32_t sb[16];
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4) {
                            const float4 gm = g4[8 * qt + q4];
                            uint32_t *y = sv + 4 * q4;
                            const float2 s01 = make_float2(__uint_as_float(y[0]), __uint_as_float(y[1]));
                            const float2 s23 = make_float2(__uint_as_float(y[2]), __uint_as_float(y[3]));
                            sb[2 * q4] = pack_bf16(s01.x, s01.y);
                            sb[2 * q4 + 1] = pack_bf16(s23.x, s23.y);
                            const float2 g01 = fmul2(make_float2(gm.x, gm.y), s01);
                            const float2 g23 = fmul2(make_float2(gm.z, gm.w), s23);
                            y[0] = __float_as_uint(g01.x);
                            y[1] = __float_as_uint(g01.y);
                            y[2] = __float_as_uint(g23.x);
                            y[3] = __float_as_uint(g23.y);
                        }
                        tmem_st16(tm + la + COL_S16 + 16 * qt, sb);
                        tmem_st16(tm + la + COL_S + 32 * qt, *reinterpret_cast<uint32_t(*)[16]>(sv));
                        tmem_st16(tm + la + COL_S + 32 * qt + 16, *reinterpret_cast<uint32_t(*)[16]>(sv + 16));
                        if (tid == 0) KDA_TR(qt == 1 ? TR_S_H0 : TR_S_H1, c);
                    } else if (ch.hT) {
                        OutRegs srr;
#pragma unroll
                        for (int i = 0; i < 32; ++i) srr.v[i] = sv[i];
                        store_state_quarter(ch.hT + (size_t)(32 * qt) * kD + j, srr);
                    }
                }
                tmem_wait_ld();
                if (tid == 0) KDA_TR(TR_S_OLD, c);
                if (ready) o_step = c;
                tmem_wait_st();
                tc_fence_before();
                if (tid == 0) bars.stop[kPrep] = *abortp;
                group_sync(1);
                if (tid == 0) KDA_TR(TR_SCAN_READY, c);
            } else {
                fail(bars);
                tc_fence_before();
                if (tid == 0) bars.stop[kPrep] = 1;
                group_sync(1);
            }
            alive = bars.stop[kPrep] == 0;
        }
        // outputs still pending: the staged step and the last step
        if (o_issuer) bulk_wait_group_read<0>();
        group_sync(1);
        if (!*abortp) flush_o();
        store_o();
        group_sync(1);
        if (!*abortp) flush_o();
        if (o_issuer) bulk_wait_group<0>();
        if (tid == 0 && issued) {
            tc_commit(&bars.drain_scan);
            mbar_wait_drain(&bars.drain_scan, 0, kWaitLimit);
        }
        if (loader) {
            // every requested tile must have landed before the CTA exits
            for (int s = loads - kSlots < 0 ? 0 : loads - kSlots; s < loads; ++s)
                mbar_wait_drain(&bars.slot_full[s % kSlots], (s / kSlots) & 1, kWaitLimit);
        }
    } else {
        // ================================================ prep warpgroups
        const int pg = (warp - 4) >> 2;                 // steps pg, pg + kPrep, ...
        const int pw = warp & 3;                        // TMEM lane quarter
        const int pt = tid - 128 - 128 * pg;
        const int bar_id = 2 + pg;
        // serial roles on different SM sub-partitions (warp w runs on w % 4;
        // the scan issuer is warp 0)
        const int iss_w = 1 + (pg + 1) % 3;             // 2, 3, 1
        const int solve_w = 1 + pg;                     // 1, 2, 3
        const bool iss = pw == iss_w && lane == 0;
        unsigned char *scr = sm + SM_SC + pg * kScBytes;
        const uint32_t scr_u = s_base + SM_SC + pg * kScBytes;
        float *dlt = reinterpret_cast<float *>(sm + SM_DELTA + pg * 512);
        const uint32_t tP = tm + COL_PREP + 64 * pg;
        const uint32_t tPl = tP + ((uint32_t)(32 * pw) << 16);
        bool issued = false;
        constexpr uint32_t idA = idesc_bf16(128, 32, false, false);
        constexpr uint32_t idZ = idesc_bf16(128, 32, true, false);

        // beta of this warpgroup's next step, loaded one step ahead (warp 0)
        auto load_beta = [&](int s) {
            const int Ls = min(kStep, L - kStep * s);
            const int64_t tok = start + (int64_t)kStep * s + lane;
            return lane < Ls ? __bfloat162float(p.beta[(size_t)tok * p.H + h]) : 0.f;
        };
        float beta_pre = (pw == 0 && pg < nS) ? load_beta(pg) : 0.f;

        for (int s = pg, u = 0; s < nS; s += kPrep, ++u) {
            const int sl = s % kSlots;
            unsigned char *slot = sm + SM_SLOT + sl * kSlotBytes;
            const uint32_t slot_u = s_base + SM_SLOT + sl * kSlotBytes;
            const int Ls = min(kStep, L - kStep * s);
            const uint32_t par = u & 1;
            if (pw == 0) {
                bars.beta_s[pg][lane] = beta_pre;
                if (s + kPrep < nS) beta_pre = load_beta(s + kPrep);
            }
            bool ok = warp_wait(&bars.slot_full[sl], (s / kSlots) & 1, abortp, p.wait_limit);
            if (!ok) fail(bars);
            if (ok && pt == 0) KDA_TR(TR_PREP_FULL, s);

            // ---------------- gate, decay and scaled operands (in place)
            if (ok) {
                float *eps_out = reinterpret_cast<float *>(sm + SM_EPS + sl * 512);
                if (Ls == kStep) gate_pass<true>(slot, pw, lane, Ls, eps_out, dlt);
                else gate_pass_partial(slot, pw, lane, Ls, eps_out, dlt);
            }
            fence_proxy_async_smem();
            group_sync(bar_id);                                             // operands written
            if (kProbe && s == p.range_step && blockIdx.x == 0) range_probe_operands(slot, pt);

            // ---------------- A_kk (TMEM lanes 0-31) and A_qk (lanes 32-63)
            if (iss && !*abortp) {
                KDA_TR(TR_PREP_P1, s);
                tc_fence_after();
                const uint64_t da = sdesc(slot_u, 16, 1024, kLayoutSW128);
                const uint64_t dg = sdesc(slot_u + SL_G0, 16, 1024, kLayoutSW128);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tP, sdesc_at(da, (kk >> 2) * SL_K1 + (kk & 3) * 32),
                           sdesc_at(dg, (kk >> 2) * (SL_G1 - SL_G0) + (kk & 3) * 32), idA, kk > 0);
                tc_commit(&bars.a_done[pg]);
                issued = true;
            }
            if (pw >= 2) {
                // step decay gamma = eps * delta, for the scan warpgroup
                if (ok) {
                    const int c2 = 2 * (pt - 64);
                    const float2 e2 = *reinterpret_cast<const float2 *>(sm + SM_EPS + sl * 512 + 4 * c2);
                    const float2 d2 = *reinterpret_cast<const float2 *>(dlt + c2);
                    *reinterpret_cast<float2 *>(sm + SM_GAMMA + sl * 512 + 4 * c2) = fmul2(e2, d2);
                }
            } else {
                // warp 0: (Diag(beta) strict_lower(A_kk))^T; warp 1: causal(A_qk)
                if (warp_wait(&bars.a_done[pg], par, abortp, p.wait_limit)) {
                    if (pt == 0) KDA_TR(TR_PREP_A, s);
                    tc_fence_after();
                    const int r = lane;
                    const float bl = bars.beta_s[pg][r];
                    float *at = reinterpret_cast<float *>(scr + SC_AT);
#pragma unroll 1
                    for (int kg = 0; kg < 4; ++kg) {
                        uint32_t d[8];
                        tmem_ld8(tPl + 8 * kg, d);
                        tmem_wait_ld();
                        if (pw == 0) {
#pragma unroll
                            for (int t = 0; t < 8; ++t) {
                                const int i = 8 * kg + t;
                                at[i * (kScRow / 4) + r] = i < r ? bl * __uint_as_float(d[t]) : 0.f;
                            }
                        } else {
                            float x[8];
#pragma unroll
                            for (int t = 0; t < 8; ++t) {
                                const int i = 8 * kg + t;
                                x[t] = i <= r ? __uint_as_float(d[t]) : 0.f;
                            }
                            uint4 w;
                            w.x = pack_bf16(x[0], x[1]);
                            w.y = pack_bf16(x[2], x[3]);
                            w.z = pack_bf16(x[4], x[5]);
                            w.w = pack_bf16(x[6], x[7]);
                            *reinterpret_cast<uint4 *>(scr + SC_AQ + core32_off(r, 8 * kg)) = w;
                        }
                    }
                } else {
                    fail(bars);
                    ok = false;
                }
                tc_fence_before();
            }
            group_sync(bar_id);                                             // scratch written

            // ---------------- T = M^-1 Diag(beta), M = I + N, N = Diag(beta) strict_lower(A_kk),
            // by 16 x 16 blocks: M = [M11 0 ; M21 M22], T11 = M11^-1 D1, T22 = M22^-1 D2,
            // T21 = -M22^-1 (M21 T11).  The scratch at[i][r] = N[r][i] (36-float rows)
            // also holds the blocks, each where a finished stage no longer reads:
            //   T11 in at[0..15][0..15], M22^-1 in at[16..31][0..15] (after stage 1),
            //   Y = M21 T11 in at[16..31][16..31] (stage 2), T21 in at[0..15][16..31] (stage 3).
            constexpr int kRs = kScRow / 4;
            float *at = reinterpret_cast<float *>(scr + SC_AT);
            float tcol[kTile];
            // (1) solver warp, lane = column: lanes 0-15 invert M11, lanes 16-31 M22
            //     (right-looking forward substitution inside the block)
            if (pw == solve_w && !*abortp) {
                const int b0 = lane & 16, cc = lane & 15;
                float acc[kTile];
#pragma unroll
                for (int r = 0; r < kTile; ++r) acc[r] = 0.f;
#pragma unroll
                for (int i = 0; i < kTile; ++i) {
                    tcol[i] = (i == cc ? 1.f : 0.f) - acc[i];
#pragma unroll
                    for (int r4 = (i + 1) & ~3; r4 < kTile; r4 += 4) {
                        const float4 a = *reinterpret_cast<const float4 *>(at + (b0 + i) * kRs + b0 + r4);
                        if (r4 > i) acc[r4] = fmaf(a.x, tcol[i], acc[r4]);
                        if (r4 + 1 > i) acc[r4 + 1] = fmaf(a.y, tcol[i], acc[r4 + 1]);
                        if (r4 + 2 > i) acc[r4 + 2] = fmaf(a.z, tcol[i], acc[r4 + 2]);
                        if (r4 + 3 > i) acc[r4 + 3] = fmaf(a.w, tcol[i], acc[r4 + 3]);
                    }
                }
                __syncwarp();
                // column cc of M_bb^-1: T11 = M11^-1 D1 (lanes 0-15), M22^-1 (lanes 16-31);
                // tcol becomes the column of T_bb
                const float bc = bars.beta_s[pg][lane];
#pragma unroll
                for (int r = 0; r < kTile; ++r) {
                    at[(b0 + r) * kRs + cc] = b0 ? tcol[r] : tcol[r] * bc;
                    tcol[r] *= bc;
                }
            }
            group_sync(bar_id);
            // (2) all threads: Y = M21 T11, two entries each (M21[r][k] = N[16 + r][k] = at[k][16 + r])
            if (!*abortp) {
                const int r = pt >> 3, c = 2 * (pt & 7);
                float2 y = make_float2(0.f, 0.f);
#pragma unroll
                for (int k = 0; k < kTile; ++k) {
                    const float m = at[k * kRs + kTile + r];
                    y = ffma2(make_float2(m, m), *reinterpret_cast<const float2 *>(at + k * kRs + c), y);
                }
                *reinterpret_cast<float2 *>(at + (kTile + r) * kRs + kTile + c) = y;
            }
            group_sync(bar_id);
            // (3) T21 = -M22^-1 Y (M22^-1 is unit lower triangular)
            if (!*abortp) {
                const int r = pt >> 3, c = 2 * (pt & 7);
                float2 t = make_float2(0.f, 0.f);
#pragma unroll
                for (int k = 0; k < kTile; ++k)
                    if (k <= r) {
                        const float u = -at[(kTile + r) * kRs + k];
                        t = ffma2(make_float2(u, u),
                                  *reinterpret_cast<const float2 *>(at + (kTile + k) * kRs + kTile + c), t);
                    }
                *reinterpret_cast<float2 *>(at + r * kRs + kTile + c) = t;
            }
            group_sync(bar_id);
            // (4) solver warp: T bf16, row c = column c of T (B operand of the Z and P
            //     products): [T11 col | T21 col] for c < 16, [0 | T22 col] for c >= 16
            if (pw == solve_w && !*abortp) {
                const bool lo = lane < 16;
                float hi[kTile];
#pragma unroll
                for (int r = 0; r < kTile; ++r) hi[r] = lo ? at[r * kRs + kTile + lane] : tcol[r];
#pragma unroll
                for (int kg = 0; kg < 2; ++kg) {
                    uint4 w;
                    w.x = lo ? pack_bf16(tcol[8 * kg], tcol[8 * kg + 1]) : 0u;
                    w.y = lo ? pack_bf16(tcol[8 * kg + 2], tcol[8 * kg + 3]) : 0u;
                    w.z = lo ? pack_bf16(tcol[8 * kg + 4], tcol[8 * kg + 5]) : 0u;
                    w.w = lo ? pack_bf16(tcol[8 * kg + 6], tcol[8 * kg + 7]) : 0u;
                    *reinterpret_cast<uint4 *>(scr + SC_TB + core32_off(lane, 8 * kg)) = w;
                    uint4 v;
                    v.x = pack_bf16(hi[8 * kg], hi[8 * kg + 1]);
                    v.y = pack_bf16(hi[8 * kg + 2], hi[8 * kg + 3]);
                    v.z = pack_bf16(hi[8 * kg + 4], hi[8 * kg + 5]);
                    v.w = pack_bf16(hi[8 * kg + 6], hi[8 * kg + 7]);
                    *reinterpret_cast<uint4 *>(scr + SC_TB + core32_off(lane, 16 + 8 * kg)) = v;
                }
                fence_proxy_async_smem();
            }
            group_sync(bar_id);                                             // T written

            // ---------------- Z = Kh^T T (cols 0-31) and P = causal(A_qk) T (cols 32-63)
            if (iss && !*abortp) {
                KDA_TR(TR_PREP_T, s);
                tc_fence_after();
                const uint64_t dh = sdesc(slot_u + SL_G0, SL_G1 - SL_G0, 1024, kLayoutSW128);
                const uint64_t dt = sdesc(scr_u + SC_TB, 128, 512, kLayoutNone);
                const uint64_t dq = sdesc(scr_u + SC_AQ, 128, 512, kLayoutNone);
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                    mma_ss(tP, sdesc_at(dh, 2048 * kk), sdesc_at(dt, 256 * kk), idZ, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                    mma_ss(tP + 32, sdesc_at(dq, 256 * kk), sdesc_at(dt, 256 * kk), idA, kk > 0);
                tc_commit(&bars.z_done[pg]);
            }
            // ---------------- Ke = Kr Diag(eps), Qe = Qr Diag(eps) in place (the A_kk /
            // A_qk product has read Kr and Qr; the Z and P products do not use them)
            if (!*abortp) {
                const int kb = pw & 1, cc = 2 * lane, r0 = 16 * (pw >> 1);
                const float2 ep = *reinterpret_cast<const float2 *>(sm + SM_EPS + sl * 512 + 4 * (64 * kb + cc));
                unsigned char *tk = slot + (kb ? SL_K1 : SL_K0), *tq = slot + (kb ? SL_Q1 : SL_Q0);
                const uint32_t cbase = (uint32_t)r0 * 128u + (uint32_t)(lane & 3) * 4u;
                const uint32_t chunk = (uint32_t)(lane >> 2);
#pragma unroll 8
                for (int rr = 0; rr < kTile; ++rr) {
                    const uint32_t o = cbase + (rr >> 3) * 1024u + (rr & 7) * 128u + ((chunk ^ (rr & 7)) << 4);
                    const float2 kv = fmul2(bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(tk + o)), ep);
                    const float2 qv = fmul2(bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(tq + o)), ep);
                    *reinterpret_cast<uint32_t *>(tk + o) = pack_bf16(kv.x, kv.y);
                    *reinterpret_cast<uint32_t *>(tq + o) = pack_bf16(qv.x, qv.y);
                }
            }
            // ---------------- [P ; Diag(delta) Z]: operand B of MMA2
            if (warp_wait(&bars.z_done[pg], par, abortp, p.wait_limit)) {
                if (pt == 0) KDA_TR(TR_PREP_Z, s);
                tc_fence_after();
                uint32_t zv[32];
                tmem_ld32(tPl, zv);
                tmem_wait_ld();
                if (kProbe && s == p.range_step && blockIdx.x == 0) {
                    OutRegs zr;
#pragma unroll
                    for (int c2 = 0; c2 < kStep; ++c2) zr.v[c2] = zv[c2];
                    range_probe_z(zr);
                }
                const int i = 32 * pw + lane;           // key channel
                const float di = dlt[i];
#pragma unroll
                for (int kg = 0; kg < 4; ++kg) {
                    uint4 w;
                    w.x = pack_bf16(di * __uint_as_float(zv[8 * kg]), di * __uint_as_float(zv[8 * kg + 1]));
                    w.y = pack_bf16(di * __uint_as_float(zv[8 * kg + 2]), di * __uint_as_float(zv[8 * kg + 3]));
                    w.z = pack_bf16(di * __uint_as_float(zv[8 * kg + 4]), di * __uint_as_float(zv[8 * kg + 5]));
                    w.w = pack_bf16(di * __uint_as_float(zv[8 * kg + 6]), di * __uint_as_float(zv[8 * kg + 7]));
                    *reinterpret_cast<uint4 *>(slot + SL_B2 + core32_off(32 + i, 8 * kg)) = w;
                }
                if (pw == 0) {                          // lanes 0-31 hold the rows of P
                    uint32_t pv[32];
                    tmem_ld32(tPl + 32, pv);
                    tmem_wait_ld();
#pragma unroll
                    for (int kg = 0; kg < 4; ++kg) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(pv[8 * kg]), __uint_as_float(pv[8 * kg + 1]));
                        w.y = pack_bf16(__uint_as_float(pv[8 * kg + 2]), __uint_as_float(pv[8 * kg + 3]));
                        w.z = pack_bf16(__uint_as_float(pv[8 * kg + 4]), __uint_as_float(pv[8 * kg + 5]));
                        w.w = pack_bf16(__uint_as_float(pv[8 * kg + 6]), __uint_as_float(pv[8 * kg + 7]));
                        *reinterpret_cast<uint4 *>(slot + SL_B2 + core32_off(lane, 8 * kg)) = w;
                    }
                }
            } else {
                fail(bars);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            if (pt == 0) bars.stop[pg] = *abortp;
            group_sync(bar_id);                                             // [P ; Z] written
            if (pt == 0 && bars.stop[pg] == 0) {
                mbar_arrive(&bars.b_ready[pg]);
                KDA_TR(TR_PREP_B, s);
            }
            if (bars.stop[pg]) break;
        }
        if (iss && issued) {
            tc_commit(&bars.drain_prep[pg]);
            mbar_wait_drain(&bars.drain_prep[pg], 0, kWaitLimit);
        }

    }

    tc_fence_before();
    __syncwarp();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tm, kTmemCols);
#ifdef KDA_TRACE
    if (tid == 0 && blockIdx.x < 1024) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        g_cta_time[blockIdx.x][1] = t;
    }
#endif
}

// Segment combine: for each head, S_{s+1} = M_s S_s + R_s for s = 1 .. G-1, in
// fp32, starting from S_1 (the final state of segment 0's run); S_G is the
// final state (hT).  One CTA per head; the running state and the current
// transfer matrix sit in shared memory (128 KB).
__global__ void __launch_bounds__(256)
seg_combine_kernel(const float *__restrict__ M, const float *__restrict__ R,
                   float *__restrict__ S, float *__restrict__ hT, const int32_t *__restrict__ cu,
                   long T, int H, int G) {
    // malformed bounds (reported by the local pass): the states were never
    // written, so nothing is combined
    if (cu != nullptr && (cu[0] != 0 || (long)cu[1] != T)) return;
    extern __shared__ __align__(16) float shm[];
    float *Sc = shm;               // [128][128]
    float *Ms = shm + kD * kD;     // [128][128]
    const int h = blockIdx.x, t = threadIdx.x;
    constexpr size_t kSt = (size_t)kD * kD;
    for (int e = t; e < kD * kD; e += 256) Sc[e] = S[((size_t)1 * H + h) * kSt + e];
    const int j = t & (kD - 1), i0 = t >> 7;     // column j, rows i0 + 2m
    for (int s = 1; s <= G - 1; ++s) {
        __syncthreads();
        const float *Mg = M + ((size_t)s * H + h) * kSt;
        for (int e = t; e < kD * kD; e += 256) Ms[e] = Mg[e];
        __syncthreads();
        const float *Rg = R + ((size_t)s * H + h) * kSt;
        float acc[kD / 2];
#pragma unroll
        for (int m = 0; m < kD / 2; ++m) acc[m] = Rg[(size_t)(i0 + 2 * m) * kD + j];
        for (int k = 0; k < kD; ++k) {
            const float skj = Sc[k * kD + j];
#pragma unroll
            for (int m = 0; m < kD / 2; ++m) acc[m] = fmaf(Ms[(i0 + 2 * m) * kD + k], skj, acc[m]);
        }
        __syncthreads();
        // start state of segment s + 1, or the final state after the last one
        float *Sg = s + 1 < G ? S + ((size_t)(s + 1) * H + h) * kSt : (hT ? hT + (size_t)h * kSt : nullptr);
#pragma unroll
        for (int m = 0; m < kD / 2; ++m) {
            Sc[(i0 + 2 * m) * kD + j] = acc[m];
            if (Sg) Sg[(size_t)(i0 + 2 * m) * kD + j] = acc[m];
        }
    }
}

// Segment correction: o_t <- o_t + S_start(s)^T om_t for the tokens t of every
// segment s >= 1 (om_t = M_{s,t}^T q_t from the identity run), then the output
// gate when one is given.  Per (segment, head) this is the product
// [tokens x 128] x [128 x 128] with the start state as the right factor; it
// reads and writes each output once and is bound by HBM (about 43 flops per
// byte), so the warp-level bf16 MMA with fp32 accumulation serves.  CTA: 8
// warps, 128 tokens a tile (16 per warp), kCorTiles tiles.  The start state
// (transposed, bf16) sits in shared memory; each tile's om rows and output
// rows arrive by asynchronous 16-byte copies into one of two buffers while
// the previous tile is multiplied, so the loads overlap the math.  Rows are
// padded to 272 bytes so that each 8 x 8 matrix load touches all banks once.
constexpr int kCorThreads = 256;
constexpr int kCorTile = 128;
constexpr int kCorTiles = 8;
constexpr int kCorRow = 136;                           // bf16 per padded shared-memory row
constexpr int kCorMat = 128 * kCorRow;                 // elements of one padded 128-row matrix
constexpr int kCorSmem = 5 * kCorMat * 2;              // start state, 2 x (om tile, o tile)

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 16-byte asynchronous copy global -> shared; `bytes` 0 fills the 16 bytes
// with zeros and reads nothing.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__global__ void __launch_bounds__(kCorThreads)
seg_correct_kernel(const float *__restrict__ S, const __nv_bfloat16 *__restrict__ om,
                   __nv_bfloat16 *__restrict__ o, const __nv_bfloat16 *__restrict__ z,
                   const int32_t *__restrict__ cu, int H, long T, long seg_len, long seg0_len) {
    // malformed bounds (reported by the local pass): nothing to correct
    if (cu != nullptr && (cu[0] != 0 || (long)cu[1] != T)) return;
    extern __shared__ __align__(16) unsigned char cs_raw[];
    __nv_bfloat16 *sT = reinterpret_cast<__nv_bfloat16 *>(cs_raw);   // [n][k] = S_start[k][n]
    __nv_bfloat16 *buf = sT + kCorMat;                               // [2][om tile, o tile]
    const int sg = 1 + (int)blockIdx.z, h = (int)blockIdx.y;
    const long seg_start = seg0_len + (long)(sg - 1) * seg_len;
    const long seg_end = seg_start + seg_len < T ? seg_start + seg_len : T;
    const long t_begin = seg_start + (long)blockIdx.x * (kCorTile * kCorTiles);
    if (t_begin >= seg_end) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    long n_tiles = (seg_end - t_begin + kCorTile - 1) / kCorTile;
    if (n_tiles > kCorTiles) n_tiles = kCorTiles;
    // the om and o rows of tile `tile` into buffer `b` (rows past the segment: zeros)
    auto fetch = [&](int tile, int b) {
        const long t0 = t_begin + (long)tile * kCorTile;
        const uint32_t a_s = smem_u32(buf + (size_t)(2 * b) * kCorMat);
        const uint32_t r_s = smem_u32(buf + (size_t)(2 * b + 1) * kCorMat);
        for (int c = tid; c < kCorTile * 16; c += kCorThreads) {      // 16-byte chunks, 16 a row
            const int r = c >> 4, q = c & 15;
            const bool in = t0 + r < seg_end;
            const long t = in ? t0 + r : seg_start;                     // a valid address either way
            const uint32_t off = (uint32_t)(r * kCorRow + 8 * q) * 2u;
            cp_async16(a_s + off, om + ((size_t)(t - seg0_len) * H + h) * kD + 8 * q, in ? 16u : 0u);
            cp_async16(r_s + off, o + ((size_t)t * H + h) * kD + 8 * q, in ? 16u : 0u);
        }
        cp_async_commit();
    };
    fetch(0, 0);
    const float *Sg = S + ((size_t)sg * H + h) * kD * kD;
    for (int e = tid; e < kD * kD; e += kCorThreads)
        sT[(e & (kD - 1)) * kCorRow + (e >> 7)] = __float2bfloat16_rn(Sg[e]);
    const int g = lane >> 2, tq = lane & 3, rbase = 16 * warp;
    const uint32_t b_addr = smem_u32(sT + ((lane & 7) + (lane >> 4) * 8) * kCorRow + ((lane >> 3) & 1) * 8);
#pragma unroll 1
    for (int tile = 0; tile < (int)n_tiles; ++tile) {
        const int b = tile & 1;
        // the next tile's rows, into the other buffer (freed by the barrier that
        // closed the previous iteration)
        if (tile + 1 < (int)n_tiles) {
            fetch(tile + 1, b ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();              // this tile's rows (and the start state) are in place
        const __nv_bfloat16 *aT = buf + (size_t)(2 * b) * kCorMat;
        const __nv_bfloat16 *rT = buf + (size_t)(2 * b + 1) * kCorMat;
        const uint32_t a_addr = smem_u32(aT + (rbase + (lane & 7) + ((lane >> 3) & 1) * 8) * kCorRow +
                                         (lane >> 4) * 8);
        float acc[16][4];
#pragma unroll
        for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            uint32_t a[4];
            ldsm_x4(a, a_addr + kk * 32);
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t bb[4];
                ldsm_x4(bb, b_addr + (np * 16 * kCorRow) * 2 + kk * 32);
                mma_16816(acc[2 * np], a, bb[0], bb[1]);
                mma_16816(acc[2 * np + 1], a, bb[2], bb[3]);
            }
        }
        const long t0 = t_begin + (long)tile * kCorTile;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int r = rbase + g + 8 * hf;
            const long t = t0 + r;
            if (t >= seg_end) continue;
            __nv_bfloat16 *orow = o + ((size_t)t * H + h) * kD;
            const __nv_bfloat16 *zrow = z ? z + ((size_t)t * H + h) * kD : nullptr;
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                const int n = 8 * nt + 2 * tq;
                const float2 base = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(rT + r * kCorRow + n));
                float x0 = base.x + acc[nt][2 * hf], x1 = base.y + acc[nt][2 * hf + 1];
                if (zrow) {
                    const float2 zz = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(zrow + n));
                    x0 *= out_gate(zz.x);
                    x1 *= out_gate(zz.y);
                }
                *reinterpret_cast<__nv_bfloat162 *>(orow + n) = __floats2bfloat162_rn(x0, x1);
            }
        }
        __syncthreads();              // buffer b is free for the tile after next
    }
}

}  // namespace prefill

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// [T_tot, H, 128] bf16 viewed as 3-D (128, H, T_tot); box (64, 1, 32), 128B swizzle.
inline bool make_qkvg_map(CUtensorMap *map, const void *base, int H, int64_t T_tot) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)T_tot};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)H * 128 * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)prefill::kBatchTok};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// SM count of the current device, looked up once per device.
inline int sm_count() {
    constexpr int kMaxDev = 64;
    static std::atomic<int> cache[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    int n = (dev >= 0 && dev < kMaxDev) ? cache[dev].load(std::memory_order_relaxed) : 0;
    if (n == 0) {
        int v = 0;
        n = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0
                ? v
                : 148;
        if (dev >= 0 && dev < kMaxDev) cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// How a single long sequence per head is split into segments (G = 1: not
// split).  Cost model in waves of one-chain-per-SM CTAs: the local pass runs
// H*(2G-1) chains and the final pass H*(G-1), each over T/G tokens.
struct SegPlan {
    int G;
    long seg_len;      // segments 1 .. G-1
    long seg0_len;     // segment 0: a whole multiple of seg_len
};

// Segments for one long sequence per head.  The local pass is the only pass
// of serial chains: segment 0 (final after it) and, for each later segment,
// one run from zero and one from the identity; the combine and the correction
// after it are short.  Segment 0 may be k times as long as the others: its H
// runs start first on H SMs while the other SMs work through the 2 H (G - 1)
// short runs, which can even out the local pass's last wave.  Cost model, in
// units of one short run: k + ceil(r / sms) with r the short runs left after
// k of them per free SM (or ceil(n / (sms - H)) when none are left); the plan
// minimises it per token of the sequence, and among equal costs keeps the
// fewest segments (a shorter combine, fewer CTAs).
inline SegPlan plan_segments(int N, int64_t T, int H) {
    SegPlan pl{1, (long)T, (long)T};
    if (N != 1 || T < 8192) return pl;
    const int sms = sm_count();
    double best = (double)((H + sms - 1) / sms);
    for (int G = 2; G <= 64; ++G) {
        for (int k = 1; k <= 3; ++k) {
            const long seg = (long)(((T + (k + G - 1) - 1) / (k + G - 1) + 31) / 32 * 32);
            if (seg < 4096) continue;
            const long seg0 = (long)k * seg;
            const int64_t last = T - seg0 - (int64_t)(G - 2) * seg;      // length of segment G - 1
            if (last <= 0 || last > seg) continue;
            const long n = 2L * H * (G - 1);
            double local;
            if (H >= sms) {
                local = (double)((H * (long)k + n + sms - 1) / sms);
            } else {
                const long early = (long)k * (sms - H);
                const long r = n > early ? n - early : 0;
                local = r > 0 ? (double)k + (double)((r + sms - 1) / sms)
                              : (double)std::max<long>(k, (n + (sms - H) - 1) / (sms - H));
            }
            const double cost = local * (double)seg / (double)T;
            if (cost < 0.97 * best) {
                best = cost;
                pl = SegPlan{G, seg, seg0};
            }
        }
    }
    return pl;
}

// One-shot diagnostic (kda_debug_stall_prefill): the next tensor-core
// prefill call makes every CTA's scan wait, at step `step`, on a barrier that
// nothing arrives on, with a bound of `limit` cycles.
struct DebugRange {
    std::atomic<int> step{-1};
};
inline DebugRange &debug_range() {
    static DebugRange d;
    return d;
}

struct DebugStall {
    std::atomic<int> step{-1};
    std::atomic<unsigned long long> limit{0};
};
inline DebugStall &debug_stall() {
    static DebugStall d;
    return d;
}

// Segmented runs: R, M and S states (3 x G x H fp32 128 x 128), then the
// identity runs' outputs for the tokens after segment 0 (bf16).
inline size_t sm100_workspace_bytes(int N, int64_t T, int H) {
    const SegPlan pl = plan_segments(N, T, H);
    if (pl.G <= 1) return 0;
    return 3 * (size_t)pl.G * H * prefill::kD * prefill::kD * sizeof(float) +
           (size_t)(T - pl.seg0_len) * H * prefill::kD * sizeof(__nv_bfloat16);
}

inline kda_status sm100_chunk_fwd(const void *q, const void *k, const void *v, const void *g,
                                  const void *beta, const float *h0, const int32_t *cu, int N,
                                  int64_t T_tot, int H, const void *z, void *o, float *hT,
                                  void *workspace, cudaStream_t s) {
    CUtensorMap mq, mk, mv, mg, mo, mom;
    // With no tokens the token pointers may be NULL and no tile is ever
    // copied (every chain is empty, or malformed and skipped); the maps then
    // describe one row of hT, which the caller passes whenever this runs.
    const int64_t T_map = T_tot > 0 ? T_tot : 1;
    auto base = [&](const void *ptr) { return T_tot > 0 ? ptr : static_cast<const void *>(hT); };
    if (!make_qkvg_map(&mq, base(q), H, T_map) || !make_qkvg_map(&mk, base(k), H, T_map) ||
        !make_qkvg_map(&mv, base(v), H, T_map) || !make_qkvg_map(&mg, base(g), H, T_map) ||
        !make_qkvg_map(&mo, base(o), H, T_map))
        return KDA_ERR_CUDA;
    const int range_step = debug_range().step.exchange(-1);
    auto kern = z ? prefill::chunk_fwd_sm100_kernel<true>
                  : (range_step >= 0 ? prefill::chunk_fwd_sm100_kernel<false, true>
                                     : prefill::chunk_fwd_sm100_kernel<false>);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)prefill::kSmemAlloc) != cudaSuccess)
        return KDA_ERR_CUDA;
    prefill::Params p;
    p.beta = static_cast<const __nv_bfloat16 *>(beta);
    p.z = static_cast<const __nv_bfloat16 *>(z);
    p.h0 = h0;
    p.cu = cu;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.hT = hT;
    p.N = N;
    p.H = H;
    p.T_tot = (long)T_tot;
    p.mode = prefill::kModeChains;
    p.G = 1;
    p.seg_len = (long)T_tot;
    p.seg0_len = (long)T_tot;
    p.ws_R = p.ws_M = p.ws_S = nullptr;
    p.om = nullptr;
    p.stall_step = debug_stall().step.exchange(-1);
    p.range_step = range_step;
    const unsigned long long lim = debug_stall().limit.exchange(0);
    p.wait_limit = (p.stall_step >= 0 && lim > 0) ? lim : prefill::kWaitLimit;
    const SegPlan pl = plan_segments(N, T_tot, H);
    if (pl.G <= 1) {
        kern<<<(unsigned)(N * H), prefill::kThreads, prefill::kSmemAlloc, s>>>(mq, mk, mv, mg, mo, mo, p);
        return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    // one long sequence per head: local pass, combine, correction
    const size_t per = (size_t)pl.G * H * prefill::kD * prefill::kD;
    float *ws = static_cast<float *>(workspace);
    p.G = pl.G;
    p.seg_len = pl.seg_len;
    p.seg0_len = pl.seg0_len;
    p.ws_R = ws;
    p.ws_M = ws + per;
    p.ws_S = ws + 2 * per;
    p.om = reinterpret_cast<__nv_bfloat16 *>(ws + 3 * per);
    if (!make_qkvg_map(&mom, p.om, H, T_tot - pl.seg0_len)) return KDA_ERR_CUDA;
    p.mode = prefill::kModeSegLocal;
    kern<<<(unsigned)(H * (2 * pl.G - 1)), prefill::kThreads, prefill::kSmemAlloc, s>>>(mq, mk, mv, mg, mo, mom, p);
    if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    const int comb_smem = 2 * prefill::kD * prefill::kD * (int)sizeof(float);
    if (cudaFuncSetAttribute(prefill::seg_combine_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, comb_smem) != cudaSuccess)
        return KDA_ERR_CUDA;
    prefill::seg_combine_kernel<<<(unsigned)H, 256, comb_smem, s>>>(p.ws_M, p.ws_R, p.ws_S, hT, cu,
                                                                   (long)T_tot, H, pl.G);
    if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    if (cudaFuncSetAttribute(prefill::seg_correct_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             prefill::kCorSmem) != cudaSuccess)
        return KDA_ERR_CUDA;
    const long per_cta = (long)prefill::kCorTile * prefill::kCorTiles;
    const dim3 cgrid((unsigned)((pl.seg_len + per_cta - 1) / per_cta), (unsigned)H, (unsigned)(pl.G - 1));
    prefill::seg_correct_kernel<<<cgrid, prefill::kCorThreads, prefill::kCorSmem, s>>>(
        p.ws_S, p.om, static_cast<__nv_bfloat16 *>(o), static_cast<const __nv_bfloat16 *>(z), cu, H,
        (long)T_tot, pl.seg_len, pl.seg0_len);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace kda
