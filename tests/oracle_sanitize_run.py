"""Calls every entry point of the CPU oracle on small and ragged inputs, with
the oracle library given on the command line (a build with AddressSanitizer
and UndefinedBehaviorSanitizer, see tests/test_oracle_sanitized.py). Checks
nothing itself: the sanitizers abort the process on an out-of-bounds access,
a use after free or undefined behaviour, and the test reads the exit status.
Prints "done" when every call returned. With --pins it runs the oracle's pin
suite (tests/test_oracle_pins.py) on the same library instead, except the
comparison with Triton's Philox, which runs in an interpreter of its own."""
import sys
from pathlib import Path

import numpy as np

sys.path.insert(0, str(Path(__file__).resolve().parents[1]))

import oracle  # noqa: E402
from quantized_lora_merge_b200 import workloads as wl  # noqa: E402

LIB = Path(sys.argv[1])
oracle.build = lambda force=False: LIB          # load the sanitized build instead


def bf16(x):
    return wl.to_bf16_bits(np.asarray(x, np.float32))


def main():
    rng = np.random.default_rng(99)
    oracle.philox4x32_10([1, 2, 3, 4], [5, 6])
    for e in (0, 1, 5, 2**33 + 7):
        oracle.aux_word(1, 3, e)
        for dist in range(4):
            oracle.aux_value(1, 3, e, dist)
    oracle.laplace_from_word(np.arange(0, 2**32, 2**24, dtype=np.uint64).astype(np.uint32))
    oracle.population_std(rng.normal(size=7))
    oracle.vmc_scale(0.02, 1.4, 1.5)
    for bits in (2, 4, 8):
        oracle.affine_quantize_row(rng.normal(size=5), bits)
        oracle.affine_quantize_row(np.zeros(3), bits)

    # ragged layers, both code widths, every law, row subsets
    for (d, n, r, w_bits) in [(1, 2, 1, 4), (3, 10, 2, 8), (7, 36, 5, 4), (5, 9, 3, 8)]:
        for dist in range(4):
            spec = wl.LayerSpec("t", d, n, r, w_bits, "mul", w_bits, stream_id=d + dist,
                                distribution=dist)
            W, A, B = wl.host_W(spec), wl.host_A(spec), wl.host_B(spec)
            oracle.std_f32(W)
            oracle.sigma_r(d, n, spec.seed, spec.stream_id, dist)
            oracle.aux_R(d, n, spec.seed, spec.stream_id)
            g = oracle.gen_aux(W, spec.seed, spec.stream_id, 1.5, w_bits, want_r_star=True, dist=dist)
            if d > 1:
                oracle.gen_aux(W, spec.seed, spec.stream_id, 1.5, w_bits, row_begin=1,
                               row_count=d - 1, dist=dist)
                oracle.quantize_rows(W[1:], spec.seed, spec.stream_id, g["c"], w_bits, 1, dist)
            s32 = g["s"].astype(np.float32)
            args = (g["codes"], s32, g["z"], A, B, spec.seed, spec.stream_id, g["sigma_w"],
                    g["sigma_r"], 1.5)
            oracle.mla_rows(*args, dist=dist)
            m = oracle.merge_mul(*args, w_bits, dist=dist)
            oracle.merge_shift(*args, 2 if w_bits == 4 else 4, dist=dist)
            oracle.merge_mul(*args, w_bits, row_begin=d - 1, row_count=1, dist=dist)
            oracle.merge_mul_rows(g["codes"][d - 1:], s32[d - 1:], g["z"][d - 1:], A[d - 1:], B,
                                  spec.seed, spec.stream_id, g["c"], w_bits, d - 1, dist)
            U, D = oracle.mla_rows(*args)
            oracle.shift_quantize_row(U[0], D[0], 4)

            Gb, Ab, Bb = wl.host_G_bits(spec), bf16(A), bf16(B)
            f = [wl.bf16_bits_to_f32(x).astype(np.float64) for x in (Gb, Ab, Bb)]
            oracle.ste_backward(*f)
            oracle.ste_sampled(Gb, Ab, Bb, np.array([0, d - 1]), np.array([0, n - 1]))
            oracle.ste_mask(g["codes"], g["z"])
            oracle.ste_backward_masked(*f, g["codes"], g["z"])
            oracle.ste_sampled_masked(Gb, Ab, Bb, g["codes"], g["z"], np.array([d - 1]),
                                      np.array([n - 1]))
            oracle.fakequant_bf16(m["P"], m["sbar"].astype(np.float32))

    # integer GEMM and training legs
    for planes, bound in ((1, 127), (2, 16383), (3, 2**21 - 1)):
        oracle.int_planes(bound)
        Q = rng.integers(-bound, bound + 1, size=(5, 16), dtype=np.int64)
        oracle.int_digits(Q, planes)
        X = rng.integers(-127, 128, size=(3, 16), dtype=np.int8)
        oracle.int_gemm_rows(X, np.ones(3), Q, np.ones(5))
        oracle.int_gemm_rows(X, np.ones(3), Q, np.ones(5), rows=np.array([2]))
    Xb, Wb = bf16(rng.normal(size=(4, 8))), bf16(rng.normal(size=(3, 8)))
    oracle.linear_rows(Xb, Wb)
    oracle.linear_rows(Xb, Wb, rows=np.array([3]))
    dYb, Ab, Bb = bf16(rng.normal(size=(4, 3))), bf16(rng.normal(size=(3, 2))), bf16(rng.normal(size=(2, 8)))
    oracle.train_backward(Xb, dYb, Wb, Ab, Bb)

    threads = oracle.num_threads()
    oracle.set_num_threads(1)
    oracle.set_num_threads(threads)
    print("done", flush=True)


if __name__ == "__main__":
    if "--pins" in sys.argv[2:]:
        import pytest
        # -s: a sanitizer report goes straight to stderr instead of a capture file
        sys.exit(pytest.main(["-q", "-x", "-s", "-p", "no:cacheprovider",
                              str(Path(__file__).resolve().parent / "test_oracle_pins.py"),
                              "-k", "not philox_matches_independent_implementation"]))
    main()
