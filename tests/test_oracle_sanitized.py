"""The fp64 oracle under AddressSanitizer, UndefinedBehaviorSanitizer and
LeakSanitizer (CPU only).

The oracle is the reference every GPU result is held to, so a memory error in
it (an index past a sequence's end, a state buffer too short for dk != dv, a
checkpoint slot past the last one) could make wrong values look right.  This
test compiles oracle/kda_oracle.c together with a small driver
(tests/oracle_sanitized_driver.c) with -fsanitize=address,undefined and
exact-size buffers, runs every entry point on ragged cases (an empty
sequence, a one-token sequence, lengths across the backward's 64-token
checkpoints, dk != dv in both directions, masked units, infinite gates, a
malformed cu_seqlens), and requires

  * a clean exit: no out-of-bounds access, use after free, leak or undefined
    behaviour (the sanitizers end the program with a non-zero status), and
  * results equal, element by element, to the normal -O2 build that the other
    tests load, so the instrumented run checked the same arithmetic.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
ORACLE_SRC = os.path.join(ROOT, "oracle", "kda_oracle.c")
DRIVER_SRC = os.path.join(HERE, "oracle_sanitized_driver.c")

CASES = {
    # lens, H, dk, dv, B (decode batch)
    "varlen_dv_wider": ([0, 1, 17, 40], 3, 16, 32, 2),
    "checkpoints_dk_wider": ([70, 0, 129], 2, 24, 16, 3),
}


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("asan") / "oracle_driver")
    cmd = ["gcc", "-std=c99", "-g", "-O1", "-fno-omit-frame-pointer", "-fopenmp",
           "-fsanitize=address,undefined", "-fno-sanitize-recover=all",
           "-o", exe, DRIVER_SRC, ORACLE_SRC, "-lm"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def _draw(lens, H, dk, dv, B, seed):
    rng = np.random.default_rng(seed)
    T = int(sum(lens))
    N = len(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)

    def unit_rows(shape):
        x = rng.standard_normal(shape)
        return x / np.linalg.norm(x, axis=-1, keepdims=True)

    inp = {
        "q": unit_rows((T, H, dk)), "k": unit_rows((T, H, dk)),
        "v": rng.standard_normal((T, H, dv)), "g": rng.standard_normal((T, H, dk)),
        "beta": 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H)))),
        "h0": 0.02 * rng.standard_normal((N, H, dk, dv)),
        "dO": rng.standard_normal((T, H, dv)),
        "dhT": rng.standard_normal((N, H, dk, dv)),
        "dec_q": unit_rows((B, H, dk)), "dec_k": unit_rows((B, H, dk)),
        "dec_v": rng.standard_normal((B, H, dv)), "dec_g": rng.standard_normal((B, H, dk)),
        "dec_beta": 1.0 / (1.0 + np.exp(-rng.standard_normal((B, H)))),
        "dec_S": 0.05 * rng.standard_normal((B, H, dk, dv)),
    }
    if T:
        # large and infinite gates on a few entries: forget all, keep all
        flat = inp["g"].reshape(-1)
        idx = rng.choice(flat.size, size=min(flat.size, 12), replace=False)
        flat[idx] = rng.choice([np.inf, -np.inf, 40.0, -40.0], size=idx.size)
    mask = (rng.random(N * H) < 0.5).astype(np.uint8)
    return cu, mask, inp


def _run(driver, tmp_path, lens, H, dk, dv, B, seed):
    cu, mask, inp = _draw(lens, H, dk, dv, B, seed)
    N, T = len(lens), int(cu[-1])
    d = tmp_path
    with open(d / "case.txt", "w") as f:
        f.write("%d %d %d %d %d %d\n" % (N, T, H, dk, dv, B))
        f.write(" ".join(str(int(x)) for x in cu) + "\n")
        f.write(" ".join(str(int(x)) for x in mask) + "\n")
    for name, a in inp.items():
        np.ascontiguousarray(a, dtype=np.float64).tofile(d / name)
    env = dict(os.environ, OMP_NUM_THREADS="3",
               ASAN_OPTIONS="detect_leaks=1:abort_on_error=0:exitcode=23",
               UBSAN_OPTIONS="print_stacktrace=1:halt_on_error=1")
    r = subprocess.run([driver, str(d)], capture_output=True, text=True, env=env,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-4000:]
    assert "runtime error" not in r.stderr, r.stderr[-4000:]

    def out(name, shape):
        return np.fromfile(d / name, dtype=np.float64).reshape(shape)

    return cu, mask, inp, out, [int(x) for x in open(d / "rc.txt").read().split()]


@pytest.mark.parametrize("case", sorted(CASES))
def test_oracle_clean_under_sanitizers_and_equal_to_normal_build(driver, tmp_path, case):
    lens, H, dk, dv, B = CASES[case]
    cu, mask, inp, out, rc = _run(driver, tmp_path, lens, H, dk, dv, B,
                                  seed=sorted(CASES).index(case) + 71)
    N, T = len(lens), int(cu[-1])
    # every valid call succeeds; every malformed cu_seqlens is refused
    assert rc[:6] == [0] * 6
    assert rc[6] == -1 and rc[7] == -1
    assert rc[8] == (-1 if N >= 2 else 0)

    q, k, v, g, beta = (inp[n] for n in ("q", "k", "v", "g", "beta"))
    eq = np.testing.assert_array_equal
    o, hT = oracle.forward(q, k, v, g, beta, cu, h0=inp["h0"])
    eq(out("o_sig", (T, H, dv)), o)
    eq(out("hT_sig", (N, H, dk, dv)), hT)
    o, hT = oracle.forward(q, k, v, g, beta, cu, gate="softplus")
    eq(out("o_soft", (T, H, dv)), o)
    eq(out("hT_soft", (N, H, dk, dv)), hT)

    # masked units: the same final states; skipped units are never written
    _, hT = oracle.forward(q, k, v, g, beta, cu, h0=inp["h0"],
                           unit_mask=mask.reshape(N, H).astype(bool), want_o=False)
    got = out("hT_mask", (N, H, dk, dv)).reshape(N * H, dk, dv)
    want = hT.reshape(N * H, dk, dv)
    on = mask.astype(bool)
    eq(got[on], want[on])
    assert not got[~on].any()

    names = ("dq", "dk", "dv", "dg", "dbeta", "dh0")
    shapes = {"dq": (T, H, dk), "dk": (T, H, dk), "dg": (T, H, dk), "dv": (T, H, dv),
              "dbeta": (T, H), "dh0": (N, H, dk, dv)}
    ref = oracle.backward(q, k, v, g, beta, cu, h0=inp["h0"], d_o=inp["dO"], d_hT=inp["dhT"])
    for n in names:
        eq(out("bwd_" + n, shapes[n]), ref[n])
    ref = oracle.backward(q, k, v, g, beta, cu, d_o=inp["dO"])
    for n in names:
        eq(out("bwd0_" + n, shapes[n]), ref[n])

    o, S = oracle.decode(inp["dec_q"], inp["dec_k"], inp["dec_v"], inp["dec_g"],
                         inp["dec_beta"], inp["dec_S"])
    eq(out("dec_o", (B, H, dv)), o)
    eq(out("dec_S_new", (B, H, dk, dv)), S)
