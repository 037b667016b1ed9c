// kda_chunk_sm100.cuh -- fused chunked KDA prefill on B200 tensor cores
// (bf16 inputs, fp32 state, d_k = d_v = 128, 16-token chunks).
//
// Operator (page "Kimi K3 发布核实与 Moonshot AI 主干架构演变", §3): per head
// the state S (d_k x d_v) is decayed per key channel by a_t, corrected with
// beta_t, k_t, v_t (delta rule) and read by q_t after the update; prefill uses
// a form that is recurrent across chunks and parallel inside a chunk.  Same
// page, "K3 对 Kimi Linear 的进一步修改" bullet 1: log a = -5 sigmoid(g), so the
// cumulative log-decay inside a 16-token tile stays in [-80, 0] and the
// reciprocal decay scaling fits BF16 range, letting every causal tile take
// the dense-matrix path.
//
// Chunk algorithm (16 rows r, start state S0, per key channel c):
//   e_r = exp(b_r) = prod_{i<=r} a_i,  m = b_7 (centre), eps = e^m,
//   delta = e^{b_15 - m}  (so the chunk decay is gamma = eps * delta)
//   Kr = K e^{b-m},  Qr = Q e^{b-m},  Kh = K e^{m-b}      (|exponent| <= 40)
//   A_kk = Kr Kh^T,  A_qk = Qr Kh^T
//   T = (I + Diag(beta) strict_lower(A_kk))^-1 Diag(beta)
//   W = T Kr Diag(eps),  U = T V - W S0
//   O = (Q e^b) S0 + causal(A_qk) U
//   S = Diag(delta) (Diag(eps) S0 + Kh^T U)
// On the tensor cores everything is written transposed so that the 128
// value channels are the MMA M dimension (TMEM lanes):
//   W^T = Diag(eps) Kr^T T^T      U_v^T = V^T T^T           (M=128, N=16, K=16)
//   [U | O]^T += S^T [-W ; Q e^b]^T                          (M=128, N=32, K=128)
//   O^T += U^T causal(A_qk)^T,     Y = Diag(eps)S^T... + U^T Kh   (K=16)
// The fp32 state stays in tensor memory as Y = (eps * S)^T plus the
// accumulated U^T Kh; once per chunk the scan warpgroup turns it into
// S = delta * Y, writes the bf16 copy the next chunk's MMA reads, and
// stores the next chunk's eps * S back.  The two 16x16 intra products of a
// chunk come from one M=128 MMA (K rows and Q rows of a 32-token batch
// stacked on M).
//
// CTA = one (sequence, head) chain, 416 threads:
//   warps 0-3   scan warpgroup: issues the inter-chunk MMAs, updates the
//               state, writes o and hT.
//   warps 4-7,  two intra warpgroups, alternating 32-token batches: gate,
//   warps 8-11  decay products, scaled bf16 operands, forward substitution,
//               W readback; each issues its own intra-chunk MMAs.
//   warp 12     producer: TMA loads of q, k, v, g (128B swizzle) and beta.
// Every mbarrier wait is bounded; a wait that runs out raises the device
// status word, makes the CTA drain its own copies and MMAs, free its tensor
// memory and return.
#pragma once

#include "kda_common.cuh"
#include "sm100_ptx.cuh"
#include "../../include/kda.h"

#include <cuda.h>

namespace kda {
namespace prefill {

using namespace kda::sm100;

constexpr int kC = 16;           // chunk length
constexpr int kD = 128;          // head size (d_k = d_v)
constexpr int kBatchTok = 32;    // tokens per TMA batch (two chunks)
constexpr int kRing = 6;         // chunks of scan operands in flight
constexpr int kThreads = 416;

// ---- shared memory map (offsets from a 1024-aligned base) ----
// Input slot (32 KB): eight [32 rows][64 ch] 128B-swizzled regions.  The
// intra warpgroup rewrites k and q in place with K e^{b-m} and Q e^{b-m}.
constexpr uint32_t OFF_K0 = 0, OFF_Q0 = 4096, OFF_K1 = 8192, OFF_Q1 = 12288;
constexpr uint32_t OFF_V0 = 16384, OFF_V1 = 20480, OFF_G0 = 24576, OFF_G1 = 28672;
constexpr uint32_t kSlotBytes = 32768;
constexpr uint32_t SM_RING = 2 * kSlotBytes;          // kRing x 19 KB
// Ring slot (one chunk of scan operands):
constexpr uint32_t R_B1 = 0;         // [-W ; Q e^b] 32 x 128 bf16, K-major SW128 (8 KB)
constexpr uint32_t R_KHF = 8192;     // (K e^{m-b})^T 128 x 16 fp32, K-major no-swizzle (8 KB):
                                     // channel rows, 4-token 16-byte cores, LBO 2048, SBO 128
constexpr uint32_t R_TT = 16384;     // [T ; 0] 32 x 16 bf16, no-swizzle K-major (1 KB)
constexpr uint32_t R_AQ = 17408;     // causal A_qk 16 x 16 fp32, no-swizzle K-major (1 KB)
constexpr uint32_t R_DELTA = 18432;  // e^{b_15 - m}, 128 fp32
constexpr uint32_t R_EPS = 18944;    // e^{m}, 128 fp32
constexpr uint32_t kRingBytes = 19456;
// K e^{m-b} of a 32-token batch in bf16 (both chunks, contiguous rows),
// [32][64] x 2, 128B swizzle: B operand of the A_kk/A_qk MMA.  One per
// batch of the ring.
constexpr int kKhRing = kRing / 2;
constexpr uint32_t SM_KH = SM_RING + kRing * kRingBytes;
constexpr uint32_t kKhBytes = 8192;
constexpr uint32_t kSmemBytes = SM_KH + kKhRing * kKhBytes;      // 206848
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;

// ---- tensor memory columns ----
constexpr uint32_t COL_SCR = 0;                  // 2 x 32: per intra warpgroup
constexpr uint32_t COL_RING = 64;                // kRing x 32: [U | O]^T
constexpr uint32_t COL_Y = COL_RING + 32 * kRing;    // 128: state accumulator
constexpr uint32_t COL_SBF = COL_Y + 128;        // 64: bf16 S^T (MMA A operand)
constexpr uint32_t kTmemCols = 512;
static_assert(COL_SBF + 64 <= kTmemCols, "tensor memory map overflow");

// A pipeline stage never waits more than microseconds; give up after ~2 s.
constexpr unsigned long long kWaitLimit = 1ull << 32;

#ifdef KDA_TRACE
// Stage timestamps (clock64) of the chain run by CTA 0; a profiling build only.
enum { TR_SCAN_MMA1 = 0, TR_SCAN_MMA1_DONE, TR_SCAN_MMA2, TR_SCAN_MMA2_DONE, TR_SCAN_END,
       TR_INTRA_FULL, TR_INTRA_P1, TR_INTRA_KQ, TR_INTRA_P2, TR_INTRA_W, TR_INTRA_P3,
       TR_PROD_ISSUE, TR_SCAN_OUT, TR_SCAN_RF, TR_EVENTS };
constexpr int kTraceLen = 128;
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
    uint64_t slot_full[2], slot_empty[2];
    uint64_t intra1[2], kq_done[2], intra2[2], w_done[2];
    uint64_t ring_full[kRing], ring_empty[kRing];
    uint64_t mma1_done, mma2_done, sbf_ready;
    uint64_t drain_scan, drain_intra[2];
    float beta_s[2][kBatchTok];
    uint32_t tmem_base;
    int abort_flag;
};

// Launch modes.  kModeChains: one CTA per (sequence, head).  The two
// segment modes split one long sequence per head into G segments of seg_len
// tokens (the state recurrence is linear in (S0, V), so
// S_end = M_s S_start + R_s):
//   kModeSegLocal: CTAs [0, H*G) run every segment from a zero state (the
//     real h0 for segment 0) giving R_s (segment 0's run is final: it writes
//     o and the start state of segment 1); CTAs [H*G, H*(2G-1)) run segments
//     s >= 1 with v = 0 from the identity, giving the transfer matrix M_s.
//   kModeSegFinal: CTAs [0, H*(G-1)) re-run segments s >= 1 from their true
//     start states (combined in between) and write o, and hT at the end.
enum { kModeChains = 0, kModeSegLocal = 1, kModeSegFinal = 2 };

struct Params {
    const __nv_bfloat16 *beta;
    const float *h0;
    const int32_t *cu;
    __nv_bfloat16 *o;
    float *hT;
    int N, H;
    long T_tot;
    int mode, G;
    long seg_len;
    float *ws_R, *ws_M, *ws_S;    // [G][H][128][128] each (segment modes)
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
};

__device__ __forceinline__ Chain chain_of(const Params &p, int cta) {
    Chain c;
    c.h0_identity = false;
    c.v_zero = false;
    c.write_o = true;
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
    c.ok = true;
    int s;
    if (p.mode == kModeSegLocal && cta < p.H * p.G) {
        c.h = cta / p.G;
        s = cta % p.G;
        c.h0 = (s == 0 && p.h0) ? p.h0 + (size_t)c.h * kSt : nullptr;
        c.hT = (s == 0 ? p.ws_S + ((size_t)1 * p.H + c.h) * kSt
                       : p.ws_R + ((size_t)s * p.H + c.h) * kSt);
        c.write_o = s == 0;
    } else if (p.mode == kModeSegLocal) {
        const int i = cta - p.H * p.G;
        c.h = i / (p.G - 1);
        s = 1 + i % (p.G - 1);
        c.h0 = nullptr;
        c.h0_identity = true;
        c.v_zero = true;
        c.write_o = false;
        c.hT = p.ws_M + ((size_t)s * p.H + c.h) * kSt;
    } else {
        c.h = cta / (p.G - 1);
        s = 1 + cta % (p.G - 1);
        c.h0 = p.ws_S + ((size_t)s * p.H + c.h) * kSt;
        c.hT = (s == p.G - 1 && p.hT) ? p.hT + (size_t)c.h * kSt : nullptr;
    }
    c.start = (int64_t)s * p.seg_len;
    const int64_t rem = p.T_tot - c.start;
    c.L = (int)(rem < p.seg_len ? rem : p.seg_len);
    return c;
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

// decay factor a = exp(-5 sigmoid(g)), via exp2
__device__ __forceinline__ float decay(float g) {
    return ex2(-5.0f * kLog2e * rcp(1.0f + ex2(-g * kLog2e)));
}

// Warp-uniform bounded wait: lane 0 polls, the result is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity,
                                          volatile int *abort) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, kWaitLimit);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    return ok;
}

__device__ __forceinline__ void fail(Barriers &bars) {
    bars.abort_flag = 1;
    raise_error(kErrTimeout);
}

__device__ __forceinline__ uint4 pack16(const float (&x)[kC]) {
    uint4 r;
    r.x = pack_bf16(x[0], x[1]);
    r.y = pack_bf16(x[2], x[3]);
    r.z = pack_bf16(x[4], x[5]);
    r.w = pack_bf16(x[6], x[7]);
    return r;
}

// End-of-chunk state pass of the scan warpgroup (one thread = one value
// channel = one TMEM lane): S = delta * Y, its bf16 copy for the next chunk's
// MMA, and either Y = eps_next * S for the next chunk or S itself to hT.
template <bool kNext>
__device__ __forceinline__ void state_pass(uint32_t tlane, const float4 *dl4, const float4 *ep4,
                                           float *hdst) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        uint32_t y[64];
        tmem_ld32(tlane + COL_Y + 64 * half, *reinterpret_cast<uint32_t(*)[32]>(y));
        tmem_ld32(tlane + COL_Y + 64 * half + 32, *reinterpret_cast<uint32_t(*)[32]>(y + 32));
        tmem_wait_ld();
        uint32_t sbv[32];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const float4 d = dl4[16 * half + q];
            float2 s01 = fmul2(make_float2(d.x, d.y),
                               make_float2(__uint_as_float(y[4 * q]), __uint_as_float(y[4 * q + 1])));
            float2 s23 = fmul2(make_float2(d.z, d.w),
                               make_float2(__uint_as_float(y[4 * q + 2]), __uint_as_float(y[4 * q + 3])));
            sbv[2 * q] = pack_bf16(s01.x, s01.y);
            sbv[2 * q + 1] = pack_bf16(s23.x, s23.y);
            if (kNext) {
                const float4 e = ep4[16 * half + q];
                s01 = fmul2(make_float2(e.x, e.y), s01);
                s23 = fmul2(make_float2(e.z, e.w), s23);
            }
            y[4 * q] = __float_as_uint(s01.x);
            y[4 * q + 1] = __float_as_uint(s01.y);
            y[4 * q + 2] = __float_as_uint(s23.x);
            y[4 * q + 3] = __float_as_uint(s23.y);
        }
        tmem_st16(tlane + COL_SBF + 32 * half, *reinterpret_cast<uint32_t(*)[16]>(sbv));
        tmem_st16(tlane + COL_SBF + 32 * half + 16, *reinterpret_cast<uint32_t(*)[16]>(sbv + 16));
        if (kNext) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                tmem_st16(tlane + COL_Y + 64 * half + 16 * q4, *reinterpret_cast<uint32_t(*)[16]>(y + 16 * q4));
        } else if (hdst) {
#pragma unroll
            for (int i = 0; i < 64; ++i) hdst[(size_t)(64 * half + i) * kD] = __uint_as_float(y[i]);
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_fwd_sm100_kernel(const __grid_constant__ CUtensorMap map_q,
                       const __grid_constant__ CUtensorMap map_k,
                       const __grid_constant__ CUtensorMap map_v,
                       const __grid_constant__ CUtensorMap map_g,
                       const Params p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
    const Chain ch = chain_of(p, blockIdx.x);
    const int h = ch.h;
    const int64_t start = ch.start;
    const int L = ch.L;
    const int nC = (L + kC - 1) / kC;
    const int nB = (nC + 1) / 2;

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars.slot_full[i], 2);
            mbar_init(&bars.slot_empty[i], 1);
            mbar_init(&bars.intra1[i], 4);
            mbar_init(&bars.kq_done[i], 1);
            mbar_init(&bars.intra2[i], 4);
            mbar_init(&bars.w_done[i], 1);
            mbar_init(&bars.drain_intra[i], 1);
        }
        for (int i = 0; i < kRing; ++i) {
            mbar_init(&bars.ring_full[i], 4);
            mbar_init(&bars.ring_empty[i], 4);
        }
        mbar_init(&bars.mma1_done, 1);
        mbar_init(&bars.mma2_done, 1);
        mbar_init(&bars.sbf_ready, 4);
        mbar_init(&bars.drain_scan, 1);
        bars.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&bars.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    // zero the lower half of every [T ; 0] tile (rows 16..31), once
    for (int e = tid; e < kRing * 128; e += kThreads) {
        const int s = e / 128, w = e % 128;
        reinterpret_cast<uint32_t *>(sm + SM_RING + s * kRingBytes + R_TT + 512)[w] = 0u;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = bars.tmem_base;
    const uint32_t s_base = smem_u32(sm);

    if (warp == 12) {
        // ------------------------------------------------ producer
        int last_use0 = -1, last_use1 = -1;
        if (nB > 0 && lane == 0) {
            prefetch_tmap(&map_q);
            prefetch_tmap(&map_k);
            prefetch_tmap(&map_v);
            prefetch_tmap(&map_g);
        }
        for (int b = 0; b < nB; ++b) {
            const int slot = b & 1, use = b >> 1;
            if (use > 0 && !warp_wait(&bars.slot_empty[slot], (use - 1) & 1, abortp)) {
                fail(bars);
                break;
            }
            uint64_t *full = &bars.slot_full[slot];
            if (lane == 0) {
                KDA_TR(TR_PROD_ISSUE, b);
                unsigned char *sb = sm + slot * kSlotBytes;
                mbar_expect_tx(full, ch.v_zero ? kSlotBytes - 8192 : kSlotBytes);
                const int z = (int)(start + (int64_t)b * kBatchTok);
                tma_load_3d(sb + OFF_K0, &map_k, full, 0, h, z);
                tma_load_3d(sb + OFF_K1, &map_k, full, 64, h, z);
                tma_load_3d(sb + OFF_Q0, &map_q, full, 0, h, z);
                tma_load_3d(sb + OFF_Q1, &map_q, full, 64, h, z);
                if (!ch.v_zero) {
                    tma_load_3d(sb + OFF_V0, &map_v, full, 0, h, z);
                    tma_load_3d(sb + OFF_V1, &map_v, full, 64, h, z);
                }
                tma_load_3d(sb + OFF_G0, &map_g, full, 0, h, z);
                tma_load_3d(sb + OFF_G1, &map_g, full, 64, h, z);
            }
            const int tok = b * kBatchTok + lane;
            bars.beta_s[slot][lane] =
                tok < L ? __bfloat162float(p.beta[(size_t)(start + tok) * p.H + h]) : 0.f;
            __syncwarp();
            if (lane == 0) mbar_arrive(full);
            if (slot == 0) last_use0 = use; else last_use1 = use;
        }
        // drain: every issued load must land before the CTA exits
        if (lane == 0) {
            if (last_use0 >= 0) mbar_wait(&bars.slot_full[0], last_use0 & 1, abortp, kWaitLimit);
            if (last_use1 >= 0) mbar_wait(&bars.slot_full[1], last_use1 & 1, abortp, kWaitLimit);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ intra warpgroups
        const int wg = (warp - 4) >> 2;           // 0 or 1: batches b = wg, wg + 2, ...
        const int it = tid - 128 - 128 * wg;
        const int iw = it >> 5;                   // TMEM lane quarter
        const int j = iw >> 1;                    // chunk of the batch (pass 1)
        const int kb = iw & 1;                    // 64-channel half (pass 1)
        const int cc = 2 * lane;                  // column pair inside the half
        const uint32_t offK = kb ? OFF_K1 : OFF_K0, offQ = kb ? OFF_Q1 : OFF_Q0;
        const uint32_t offV = kb ? OFF_V1 : OFF_V0, offG = kb ? OFF_G1 : OFF_G0;
        const uint32_t col_scr = COL_SCR + 32 * wg;
        const int slot = wg;
        unsigned char *sb = sm + slot * kSlotBytes;
        const uint32_t sb_u = s_base + slot * kSlotBytes;
        bool ok = true, issued = false;
        for (int kk_b = 0;; ++kk_b) {
            const int b = wg + 2 * kk_b;
            if (b >= nB) break;
            const uint32_t par = kk_b & 1;
            // ring slots for the two chunks must be free, inputs landed
            for (int jj = 0; jj < 2 && ok; ++jj) {
                const int cj = 2 * b + jj;
                if (cj < nC && cj >= kRing)
                    ok = warp_wait(&bars.ring_empty[cj % kRing], ((cj / kRing) - 1) & 1, abortp);
            }
            if (ok) ok = warp_wait(&bars.slot_full[slot], par, abortp);
            if (!ok) { fail(bars); break; }
            if (it == 0) KDA_TR(TR_INTRA_FULL, b);

            // ---------------- pass 1: gate, decay, scaled operands
            {
                const int cj = 2 * b + j;
                const bool chunk_valid = cj < nC;
                const int Lj = chunk_valid ? min(kC, L - kC * cj) : 0;
                unsigned char *ring = sm + SM_RING + (cj % kRing) * kRingBytes;
                unsigned char *khb = sm + SM_KH + (b % kKhRing) * kKhBytes;
                float2 eb[kC];                   // e^{b_r} as running products
                float2 acc = make_float2(1.f, 1.f);
                const float2 kNegLog2e = make_float2(-kLog2e, -kLog2e);
                const float2 kNeg5Log2e = make_float2(-5.f * kLog2e, -5.f * kLog2e);
                const float2 kOne = make_float2(1.f, 1.f);
#pragma unroll
                for (int r = 0; r < kC; ++r) {
                    const uint32_t o = sw128_off(16 * j + r, cc);
                    const float2 g = bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(sb + offG + o));
                    const float2 x = fmul2(g, kNegLog2e);
                    const float2 den = fadd2(make_float2(ex2(x.x), ex2(x.y)), kOne);
                    const float2 l = fmul2(make_float2(rcp(den.x), rcp(den.y)), kNeg5Log2e);
                    const float2 a = make_float2(ex2(l.x), ex2(l.y));
                    acc = fmul2(acc, (r < Lj) ? a : kOne);
                    eb[r] = acc;
                }
                const float2 em = eb[7];                                   // e^{m}
                const float2 im = make_float2(rcp(em.x), rcp(em.y));       // e^{-m}
                if (chunk_valid) {
                    float *dl = reinterpret_cast<float *>(ring + R_DELTA);
                    float *ep = reinterpret_cast<float *>(ring + R_EPS);
                    *reinterpret_cast<float2 *>(dl + 64 * kb + cc) = fmul2(eb[kC - 1], im);
                    *reinterpret_cast<float2 *>(ep + 64 * kb + cc) = em;
                }
                const int chn = 64 * kb + cc;             // first of this thread's two channels
                // (channel, token) of the fp32 K-hat tile:
                // token/4 * 2048 + channel/8 * 128 + channel%8 * 16 + token%4 * 4
                const uint32_t khf_off = R_KHF + (chn >> 3) * 128 + (chn & 7) * 16;
                float4 kq0 = make_float4(0.f, 0.f, 0.f, 0.f), kq1 = kq0;
#pragma unroll
                for (int r = 0; r < kC; ++r) {
                    const uint32_t o = sw128_off(16 * j + r, cc);
                    const bool live = r < Lj;
                    const uint32_t kraw = *reinterpret_cast<const uint32_t *>(sb + offK + o);
                    const uint32_t qraw = *reinterpret_cast<const uint32_t *>(sb + offQ + o);
                    const float2 kf = bf16x2_to_float2(live ? kraw : 0u);
                    const float2 qf = bf16x2_to_float2(live ? qraw : 0u);
                    const float2 er = fmul2(eb[r], im);                    // e^{b-m}
                    const float2 ei = make_float2(rcp(er.x), rcp(er.y));   // e^{m-b}
                    const float2 kr = fmul2(kf, er), qr = fmul2(qf, er);
                    const float2 kh = fmul2(kf, ei), qa = fmul2(qf, eb[r]);
                    *reinterpret_cast<uint32_t *>(sb + offK + o) = pack_bf16(kr.x, kr.y);
                    *reinterpret_cast<uint32_t *>(sb + offQ + o) = pack_bf16(qr.x, qr.y);
                    *reinterpret_cast<uint32_t *>(khb + kb * 4096 + sw128_off(16 * j + r, cc)) =
                        pack_bf16(kh.x, kh.y);
                    if (chunk_valid)
                        *reinterpret_cast<uint32_t *>(ring + R_B1 + kb * 4096 + sw128_off(16 + r, cc)) =
                            pack_bf16(qa.x, qa.y);
                    // four consecutive tokens of each of the two channels -> one 16-byte core row
                    if ((r & 3) == 0) { kq0.x = kh.x; kq1.x = kh.y; }
                    if ((r & 3) == 1) { kq0.y = kh.x; kq1.y = kh.y; }
                    if ((r & 3) == 2) { kq0.z = kh.x; kq1.z = kh.y; }
                    if ((r & 3) == 3) {
                        kq0.w = kh.x; kq1.w = kh.y;
                        if (chunk_valid) {
                            *reinterpret_cast<float4 *>(ring + khf_off + (r >> 2) * 2048) = kq0;
                            *reinterpret_cast<float4 *>(ring + khf_off + (r >> 2) * 2048 + 16) = kq1;
                        }
                    }
                }
                // rows past the end of the sequence (every row when v is
                // treated as zero): V must be exactly zero
                const int vz = ch.v_zero ? 0 : Lj;
                if (vz < kC)
                    for (int r = vz; r < kC; ++r)
                        *reinterpret_cast<uint32_t *>(sb + offV + sw128_off(16 * j + r, cc)) = 0u;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.intra1[wg]);
            if (it == 0) KDA_TR(TR_INTRA_P1, b);

            // ---------------- MMA: A_kk and A_qk rows of both chunks
            if (it == 0) {
                if (!mbar_wait(&bars.intra1[wg], par, abortp, kWaitLimit)) { fail(bars); ok = false; }
                else {
                    tc_fence_after();
                    constexpr uint32_t id = idesc_bf16(128, 32, false, false);
                    const uint32_t kh = s_base + SM_KH + (b % kKhRing) * kKhBytes;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t a = sdesc(sb_u + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024, kLayoutSW128);
                        const uint64_t bd = sdesc(kh + (kk >> 2) * 4096 + (kk & 3) * 32, 16, 1024, kLayoutSW128);
                        mma_ss(tm + col_scr, a, bd, id, kk > 0);
                    }
                    tc_commit(&bars.kq_done[wg]);
                    issued = true;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;

            // ---------------- pass 2: forward substitution (warp 0), causal A_qk (warp 1)
            if (iw < 2) {
                if (!warp_wait(&bars.kq_done[wg], par, abortp)) { fail(bars); ok = false; break; }
                if (it == 0) KDA_TR(TR_INTRA_KQ, b);
                tc_fence_after();
                uint32_t d[32];
                tmem_ld32(tm + ((uint32_t)(32 * iw) << 16) + col_scr, d);
                tmem_wait_ld();
                const int jj = lane >> 4, r = lane & 15;
                const int cj = 2 * b + jj;
                unsigned char *ring = sm + SM_RING + (cj % kRing) * kRingBytes;
                float X[kC];
                if (iw == 0) {
                    const float beta_l = bars.beta_s[slot][lane];
                    float A[kC];
#pragma unroll
                    for (int i = 0; i < kC; ++i) {
                        const float a = __uint_as_float(jj ? d[16 + i] : d[i]);
                        A[i] = (i < r) ? beta_l * a : 0.f;
                        X[i] = (i == r) ? beta_l : 0.f;
                    }
                    // row r of T = (I + A)^-1 Diag(beta): rows are finished in order
#pragma unroll
                    for (int i = 0; i < kC - 1; ++i) {
#pragma unroll
                        for (int col = 0; col <= i; ++col) {
                            const float t = __shfl_sync(0xffffffffu, X[col], i, 16);
                            if (r > i) X[col] = fmaf(-A[i], t, X[col]);
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < kC; ++i) {
                        const float a = __uint_as_float(jj ? d[16 + i] : d[i]);
                        X[i] = (i <= r) ? a : 0.f;
                    }
                }
                if (cj < nC) {
                    if (iw == 0) {   // T in bf16 (B operand of the W / U_v MMAs)
                        uint4 lo, hi;
                        lo.x = pack_bf16(X[0], X[1]);   lo.y = pack_bf16(X[2], X[3]);
                        lo.z = pack_bf16(X[4], X[5]);   lo.w = pack_bf16(X[6], X[7]);
                        hi.x = pack_bf16(X[8], X[9]);   hi.y = pack_bf16(X[10], X[11]);
                        hi.z = pack_bf16(X[12], X[13]); hi.w = pack_bf16(X[14], X[15]);
                        *reinterpret_cast<uint4 *>(ring + R_TT + core16_off(r, 0)) = lo;
                        *reinterpret_cast<uint4 *>(ring + R_TT + core16_off(r, 8)) = hi;
                    } else {         // causal A_qk in fp32 (B operand of the tf32 MMA)
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4)
                            *reinterpret_cast<float4 *>(ring + R_AQ + core16_off32(r, 4 * k4)) =
                                make_float4(X[4 * k4], X[4 * k4 + 1], X[4 * k4 + 2], X[4 * k4 + 3]);
                    }
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.intra2[wg]);
            if (it == 0) KDA_TR(TR_INTRA_P2, b);

            // ---------------- MMA: W^T (unscaled) and [U_v | 0]^T per chunk
            if (it == 0) {
                if (!mbar_wait(&bars.intra2[wg], par, abortp, kWaitLimit)) { fail(bars); ok = false; }
                else {
                    tc_fence_after();
                    constexpr uint32_t idw = idesc_bf16(128, 16, true, false);
                    constexpr uint32_t idu = idesc_bf16(128, 32, true, false);
                    for (int jj = 0; jj < 2; ++jj) {
                        const int cj = 2 * b + jj;
                        if (cj >= nC) break;
                        const uint32_t ring_u = s_base + SM_RING + (cj % kRing) * kRingBytes;
                        const uint64_t tdesc = sdesc(ring_u + R_TT, 128, 256, kLayoutNone);
                        mma_ss(tm + col_scr + 16 * jj,
                               sdesc(sb_u + OFF_K0 + 2048 * jj, OFF_K1 - OFF_K0, 1024, kLayoutSW128),
                               tdesc, idw, 0);
                        mma_ss(tm + COL_RING + 32 * (cj % kRing),
                               sdesc(sb_u + OFF_V0 + 2048 * jj, OFF_V1 - OFF_V0, 1024, kLayoutSW128),
                               tdesc, idu, 0);
                    }
                    tc_commit(&bars.w_done[wg]);
                    tc_commit(&bars.slot_empty[slot]);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;

            // ---------------- pass 3: -W = -(W^T * eps)^T rows of the B1 tiles
            if (!warp_wait(&bars.w_done[wg], par, abortp)) { fail(bars); ok = false; break; }
            if (it == 0) KDA_TR(TR_INTRA_W, b);
            tc_fence_after();
            {
                const int c = 32 * iw + lane;            // key channel (TMEM lane)
                const int wkb = c >> 6, wcol = c & 63;
                for (int jj = 0; jj < 2; ++jj) {
                    const int cj = 2 * b + jj;
                    if (cj >= nC) break;
                    uint32_t w[16];
                    tmem_ld16(tm + ((uint32_t)(32 * iw) << 16) + col_scr + 16 * jj, w);
                    tmem_wait_ld();
                    unsigned char *ring = sm + SM_RING + (cj % kRing) * kRingBytes;
                    const float neps = -reinterpret_cast<const float *>(ring + R_EPS)[c];
#pragma unroll
                    for (int r = 0; r < kC; ++r)
                        *reinterpret_cast<__nv_bfloat16 *>(ring + R_B1 + wkb * 4096 + sw128_off(r, wcol)) =
                            __float2bfloat16_rn(neps * __uint_as_float(w[r]));
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                for (int jj = 0; jj < 2; ++jj)
                    if (2 * b + jj < nC) mbar_arrive(&bars.ring_full[(2 * b + jj) % kRing]);
            if (it == 0) KDA_TR(TR_INTRA_P3, b);
        }
        // drain this warpgroup's MMAs before the CTA frees tensor memory
        if (it == 0 && issued) {
            tc_commit(&bars.drain_intra[wg]);
            mbar_wait(&bars.drain_intra[wg], 0, abortp, kWaitLimit);
        }
    } else {
        // ------------------------------------------------ scan warpgroup
        const int jv = tid;                               // value channel = TMEM lane
        const uint32_t lane_addr = (uint32_t)(32 * warp) << 16;
        bool ok = true, issued = false;
        const float *h0u = ch.h0 ? ch.h0 + jv : nullptr;
        if (nC > 0) {
            // initial state: bf16 copy for the first MMA, eps_0 * S0 into Y
            ok = warp_wait(&bars.ring_full[0], 0, abortp);
            if (!ok) fail(bars);
            else {
                tc_fence_after();
                const float *ep = reinterpret_cast<const float *>(sm + SM_RING + R_EPS);
#pragma unroll
                for (int part = 0; part < 4; ++part) {
                    float s0[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        s0[i] = h0u ? h0u[(size_t)(32 * part + i) * kD]
                                    : ((ch.h0_identity && 32 * part + i == jv) ? 1.f : 0.f);
                    uint32_t sb16[16], y0[16], y1[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        sb16[i] = pack_bf16(s0[2 * i], s0[2 * i + 1]);
                        y0[i] = __float_as_uint(ep[32 * part + i] * s0[i]);
                        y1[i] = __float_as_uint(ep[32 * part + 16 + i] * s0[16 + i]);
                    }
                    tmem_st16(tm + lane_addr + COL_SBF + 16 * part, sb16);
                    tmem_st16(tm + lane_addr + COL_Y + 32 * part, y0);
                    tmem_st16(tm + lane_addr + COL_Y + 32 * part + 16, y1);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.sbf_ready);
            }
        } else if (ch.hT) {
            float *dst = ch.hT + jv;
            for (int c = 0; c < kD; ++c)
                dst[(size_t)c * kD] = h0u ? h0u[(size_t)c * kD] : ((ch.h0_identity && c == jv) ? 1.f : 0.f);
        }

        for (int c = 0; c < nC && ok; ++c) {
            const int rs = c % kRing;
            const uint32_t ring_u = s_base + SM_RING + rs * kRingBytes;
            const unsigned char *ring = sm + SM_RING + rs * kRingBytes;
            const uint32_t colU = COL_RING + 32 * rs;
            // MMA1: [U | O]^T += S^T [-W ; Q e^b]^T  (bf16); then, once it has
            // landed, MMA2 reads U^T straight from tensor memory as tf32:
            // O^T += U^T causal(A_qk)^T ;  Y += U^T Kh
            if (tid == 0) {
                ok = mbar_wait(&bars.ring_full[rs], (c / kRing) & 1, abortp, kWaitLimit) &&
                     mbar_wait(&bars.sbf_ready, c & 1, abortp, kWaitLimit);
                if (ok) {
                    KDA_TR(TR_SCAN_MMA1, c);
                    tc_fence_after();
                    constexpr uint32_t id = idesc_bf16(128, 32, false, false);
                    const uint64_t b0 = sdesc(ring_u + R_B1, 16, 1024, kLayoutSW128);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts(tm + colU, tm + COL_SBF + 8 * kk,
                               b0 + (uint64_t)(((kk >> 2) * 4096 + (kk & 3) * 32) >> 4), id, 1);
                    tc_commit(&bars.mma1_done);
                    issued = true;
                    ok = mbar_wait(&bars.mma1_done, c & 1, abortp, kWaitLimit);
                }
                if (ok) {
                    KDA_TR(TR_SCAN_MMA2, c);
                    tc_fence_after();
                    constexpr uint32_t ido = idesc_tf32(128, 16, false, false);
                    constexpr uint32_t idy = idesc_tf32(128, 128, false, false);
                    const uint64_t aq = sdesc(ring_u + R_AQ, 128, 512, kLayoutNone);
                    const uint64_t kh = sdesc(ring_u + R_KHF, 2048, 128, kLayoutNone);
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        mma_ts_tf32(tm + colU + 16, tm + colU + 8 * ks, aq + (uint64_t)((256 * ks) >> 4), ido, 1);
                        mma_ts_tf32(tm + COL_Y, tm + colU + 8 * ks, kh + (uint64_t)((4096 * ks) >> 4), idy, 1);
                    }
                    tc_commit(&bars.mma2_done);
                }
                if (!ok) fail(bars);
            }
            const bool has_next = c + 1 < nC;
            if (has_next && !warp_wait(&bars.ring_full[(c + 1) % kRing], ((c + 1) / kRing) & 1, abortp)) {
                fail(bars); ok = false; break;
            }
            if (!warp_wait(&bars.mma2_done, c & 1, abortp)) { fail(bars); ok = false; break; }
            if (tid == 0) KDA_TR(TR_SCAN_MMA2_DONE, c);
            tc_fence_after();
            // this chunk's output (the tensor pipe is idle for this warpgroup now)
            uint32_t ov[16];
            tmem_ld16(tm + lane_addr + colU + 16, ov);
            // S = delta * Y  ->  bf16 copy;  Y = eps_next * S  (or hT at the end)
            {
                const float4 *dl4 = reinterpret_cast<const float4 *>(ring + R_DELTA);
                if (has_next) {
                    const float4 *ep4 = reinterpret_cast<const float4 *>(
                        sm + SM_RING + ((c + 1) % kRing) * kRingBytes + R_EPS);
                    state_pass<true>(tm + lane_addr, dl4, ep4, nullptr);
                } else {
                    float *hdst = ch.hT ? ch.hT + jv : nullptr;
                    state_pass<false>(tm + lane_addr, dl4, nullptr, hdst);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars.sbf_ready);
                mbar_arrive(&bars.ring_empty[rs]);
            }
            if (tid == 0) KDA_TR(TR_SCAN_END, c);
            if (ch.write_o) {
                const int Lc = min(kC, L - kC * c);
                __nv_bfloat16 *dst = p.o + ((size_t)(start + kC * c) * p.H + h) * kD + jv;
                const size_t step = (size_t)p.H * kD;
#pragma unroll
                for (int r = 0; r < kC; ++r)
                    if (r < Lc) dst[(size_t)r * step] = __float2bfloat16_rn(__uint_as_float(ov[r]));
            }
        }
        if (tid == 0 && issued) {
            tc_commit(&bars.drain_scan);
            mbar_wait(&bars.drain_scan, 0, abortp, kWaitLimit);
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

// Segment combine (between the two segment modes): for each head,
// S_{s+1} = M_s S_s + R_s for s = 1 .. G-2, in fp32, starting from S_1 (the
// final state of segment 0's run).  One CTA per head; the running state and
// the current transfer matrix sit in shared memory (128 KB).
__global__ void __launch_bounds__(256)
seg_combine_kernel(const float *__restrict__ M, const float *__restrict__ R,
                   float *__restrict__ S, int H, int G) {
    extern __shared__ __align__(16) float shm[];
    float *Sc = shm;               // [128][128]
    float *Ms = shm + kD * kD;     // [128][128]
    const int h = blockIdx.x, t = threadIdx.x;
    constexpr size_t kSt = (size_t)kD * kD;
    for (int e = t; e < kD * kD; e += 256) Sc[e] = S[((size_t)1 * H + h) * kSt + e];
    const int j = t & (kD - 1), i0 = t >> 7;     // column j, rows i0 + 2m
    for (int s = 1; s <= G - 2; ++s) {
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
        float *Sg = S + ((size_t)(s + 1) * H + h) * kSt;
#pragma unroll
        for (int m = 0; m < kD / 2; ++m) {
            Sc[(i0 + 2 * m) * kD + j] = acc[m];
            Sg[(size_t)(i0 + 2 * m) * kD + j] = acc[m];
        }
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

inline int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
            n = v;
        else
            n = 148;
    }
    return n;
}

// How a single long sequence per head is split into segments (G = 1: not
// split).  Cost model in waves of one-chain-per-SM CTAs: the local pass runs
// H*(2G-1) chains and the final pass H*(G-1), each over T/G tokens.
struct SegPlan {
    int G;
    long seg_len;
};

inline SegPlan plan_segments(int N, int64_t T, int H) {
    SegPlan pl{1, (long)T};
    if (N != 1 || T < 8192) return pl;
    const int sms = sm_count();
    double best = (double)((H + sms - 1) / sms);
    for (int G = 2; G <= 64; ++G) {
        const long seg = (long)(((T + G - 1) / G + 31) / 32 * 32);
        if (seg < 4096) break;
        if ((T + seg - 1) / seg != G) continue;
        const int w1 = (H * (2 * G - 1) + sms - 1) / sms;
        const int w3 = (H * (G - 1) + sms - 1) / sms;
        const double cost = (double)(w1 + w3) / G;
        if (cost < 0.9 * best) {
            best = cost;
            pl = SegPlan{G, seg};
        }
    }
    return pl;
}

inline size_t sm100_workspace_bytes(int N, int64_t T, int H) {
    const SegPlan pl = plan_segments(N, T, H);
    if (pl.G <= 1) return 0;
    return 3 * (size_t)pl.G * H * prefill::kD * prefill::kD * sizeof(float);
}

inline kda_status sm100_chunk_fwd(const void *q, const void *k, const void *v, const void *g,
                                  const void *beta, const float *h0, const int32_t *cu, int N,
                                  int64_t T_tot, int H, void *o, float *hT, void *workspace,
                                  cudaStream_t s) {
    CUtensorMap mq, mk, mv, mg;
    const int64_t T_map = T_tot > 0 ? T_tot : 1;
    if (!make_qkvg_map(&mq, q, H, T_map) || !make_qkvg_map(&mk, k, H, T_map) ||
        !make_qkvg_map(&mv, v, H, T_map) || !make_qkvg_map(&mg, g, H, T_map))
        return KDA_ERR_CUDA;
    auto kern = prefill::chunk_fwd_sm100_kernel;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)prefill::kSmemAlloc) != cudaSuccess)
        return KDA_ERR_CUDA;
    prefill::Params p;
    p.beta = static_cast<const __nv_bfloat16 *>(beta);
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
    p.ws_R = p.ws_M = p.ws_S = nullptr;
    const SegPlan pl = plan_segments(N, T_tot, H);
    if (pl.G <= 1) {
        kern<<<(unsigned)(N * H), prefill::kThreads, prefill::kSmemAlloc, s>>>(mq, mk, mv, mg, p);
        return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    // one long sequence per head: local pass, combine, final pass
    const size_t per = (size_t)pl.G * H * prefill::kD * prefill::kD;
    float *ws = static_cast<float *>(workspace);
    p.G = pl.G;
    p.seg_len = pl.seg_len;
    p.ws_R = ws;
    p.ws_M = ws + per;
    p.ws_S = ws + 2 * per;
    p.mode = prefill::kModeSegLocal;
    kern<<<(unsigned)(H * (2 * pl.G - 1)), prefill::kThreads, prefill::kSmemAlloc, s>>>(mq, mk, mv, mg, p);
    if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    const int comb_smem = 2 * prefill::kD * prefill::kD * (int)sizeof(float);
    if (cudaFuncSetAttribute(prefill::seg_combine_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, comb_smem) != cudaSuccess)
        return KDA_ERR_CUDA;
    prefill::seg_combine_kernel<<<(unsigned)H, 256, comb_smem, s>>>(p.ws_M, p.ws_R, p.ws_S, H, pl.G);
    if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    p.mode = prefill::kModeSegFinal;
    kern<<<(unsigned)(H * (pl.G - 1)), prefill::kThreads, prefill::kSmemAlloc, s>>>(mq, mk, mv, mg, p);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace kda
