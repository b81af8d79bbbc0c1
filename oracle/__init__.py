"""fp64 CPU oracle for the MXFP4 mixture-of-experts expert block.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library under
``mxfp4_quantized_moe_b200/`` and its Python binding) imports, links or runs
anything in this package.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its ``cpu_baseline`` leg and its ``--impl reference`` arm) may
call it.

Modules
-------
``mxfp4_oracle``  numpy fp64 restatement of the method: MXFP4 decode, top-k
                  routing, expert loop forward, analytic input-gradient backward.
``scalar_twin``   pure-Python loops over the same definitions, token-major and
                  without numpy linear algebra; the brute-force pin for tiny cases.
``make_golden``   the script that writes the stored expected values under
                  ``tests/golden/`` (it calls only this package).

Every function is pinned by a ``-m "not gpu"`` test (``tests/test_oracle_pins.py``)
against closed forms, invariants, brute force or finite differences.  No
function here is "parity unpinned".
"""

from .mxfp4_oracle import (  # noqa: F401
    E2M1_MAGNITUDES,
    bf16_bits_to_f64,
    dequantize,
    decode_e2m1,
    decode_ue8m0,
    f64_to_bf16_bits,
    glu,
    glu_backward,
    moe_backward,
    moe_forward,
    route,
)
