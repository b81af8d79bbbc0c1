"""Child process of tests/test_gpu_debug_build.py: runs under MXFP4_MOE_LIBRARY=debug, so the
library loaded is the debug build (device-side index checks).

1. The debug build computes the block like the library: parity against the fp64 oracle on
   small shapes (a ragged tile, a single token, most experts empty, T below the tile height).
2. An expert-sorted row whose routing slot points outside [0, T*k) is planted in the workspace
   between the forward and the backward; the debug build's dY gather records DEVICE_BOUNDS
   with its tag (0x110) instead of reading through it.  This step runs only after the library
   reported itself as the debug build.
3. The same context then computes a fresh block exactly as before.
"""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main():
    if os.environ.get("MXFP4_MOE_LIBRARY") != "debug":
        print("MXFP4_MOE_LIBRARY is not 'debug'")
        return 2
    import torch

    from mxfp4_quantized_moe_b200 import _lib, inputs, moe
    if _lib.lib.mxfp4_moe_build_flags() != 1:
        print("the loaded library is not the debug build")
        return 3
    from tests.test_gpu_parity import _ws_offsets, check_all, run_block

    # 1. parity of the debug build
    for T, H, I, E, k, seed in ((64, 256, 256, 8, 2, 0), (37, 96, 160, 5, 3, 4),
                                (5, 64, 64, 16, 1, 5), (1, 64, 64, 4, 2, 1)):
        got, ref = run_block(moe, T, H, I, E, k, seed)
        check_all(got, ref)
    print("parity ok", flush=True)

    # 2. a routing slot outside [0, T*k) planted between the forward and the backward
    T, H, I, E, k = 64, 256, 256, 8, 2
    A = T * k
    inp = inputs.make_layer(T, H, I, E, k, 3)
    shape = moe.MoeShape(T, H, I, E, k)
    w = moe.weights_to(inp, "cuda")
    ws = moe.alloc_workspace(shape)
    wt = moe.transpose_weights(shape, w)
    moe.forward(shape, w, inp["x"].cuda(), inp["logits"].cuda(), ws)
    assert moe.device_check(ws) == (0, 0)
    o = _ws_offsets(T, E, k)
    perm = ws[o["perm"]:o["perm"] + 4 * A].view(torch.int32)
    perm[3] = A + 1000
    moe.backward_input(shape, w, wt, inp["dy"].cuda(), ws)
    rc, where = moe.device_check(ws)
    assert (rc, where) == (_lib.ERR_DEVICE_BOUNDS, 0x110), (rc, hex(where))
    print("bounds check ok", flush=True)

    # 3. the context is intact
    got, ref = run_block(moe, 64, 256, 256, 8, 2, 0)
    check_all(got, ref)
    print("debug build ok", flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
