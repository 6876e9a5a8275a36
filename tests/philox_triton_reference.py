"""Independent Philox4x32-10 values from Triton's own implementation, run by
Triton's CPU interpreter (no GPU). Used only as a pin for the oracle's Philox:
the two implementations share nothing.

Usage: python philox_triton_reference.py '<json list of [c0,c1,c2,c3,k0,k1]>'
Prints a JSON list of [x0,x1,x2,x3] per case.
"""
import json
import os
import sys

os.environ["TRITON_INTERPRET"] = "1"

import torch  # noqa: E402
import triton  # noqa: E402
import triton.language as tl  # noqa: E402


@triton.jit
def _philox_kernel(c_ptr, out_ptr, seed, N: tl.constexpr):
    i = tl.arange(0, N)
    c0 = tl.load(c_ptr + 4 * i + 0)
    c1 = tl.load(c_ptr + 4 * i + 1)
    c2 = tl.load(c_ptr + 4 * i + 2)
    c3 = tl.load(c_ptr + 4 * i + 3)
    x0, x1, x2, x3 = tl.philox(seed, c0, c1, c2, c3, 10)
    tl.store(out_ptr + 4 * i + 0, x0.to(tl.int32, bitcast=True))
    tl.store(out_ptr + 4 * i + 1, x1.to(tl.int32, bitcast=True))
    tl.store(out_ptr + 4 * i + 2, x2.to(tl.int32, bitcast=True))
    tl.store(out_ptr + 4 * i + 3, x3.to(tl.int32, bitcast=True))


def main():
    cases = json.loads(sys.argv[1])
    results = []
    for c0, c1, c2, c3, k0, k1 in cases:
        seed = (k1 << 32) | k0
        ctr = torch.tensor([v - (1 << 32) if v >= (1 << 31) else v for v in (c0, c1, c2, c3)],
                           dtype=torch.int32)
        out = torch.zeros(4, dtype=torch.int32)
        # seed is a 64-bit scalar: pass it as a signed int64 value
        s = seed - (1 << 64) if seed >= (1 << 63) else seed
        _philox_kernel[(1,)](ctr, out, s, N=1)
        results.append([int(v) & 0xFFFFFFFF for v in out.tolist()])
    print(json.dumps(results))


if __name__ == "__main__":
    main()
