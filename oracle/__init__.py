"""Plain CPU oracle for the ConvRot W4A4 linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only the test suite, the smoke check in ``__graft_entry__`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may call it.  It
shares no code, tables or constants with the CUDA library; the two meet only
through the seeded input generators in ``workloads.py``, which hold none of
the method's arithmetic.

Sources (web pages on the method; cited by page title and section):
  * "[PR #63] int4_tensorwise: W4A4 layout (+ConvRot) with fused CUDA kernels"
    (comfy-kitchen issue #118), section "Description" -- the layout, the eager
    ops and the fused CUDA design.
  * "Comfy-INT4-HIPtest README", section "What it provides" -- Hadamard
    ConvRot with a configurable group size.
  * "ComfyUI-INT4-Fast Introduction" (runcomfy), section "How ComfyUI-INT4-Fast
    Works" -- what the rotation is for.
  * "Comfy-INT4-HIPtest README", section "LoRA modes", and "ComfyUI-INT4-Fast"
    (features list, "Dynamic LoRA Patching") -- the Dynamic LoRA delta, with
    the down projection rotated into the layer's basis.
Where these pages leave a constant open (the 1/sqrt(g) normalisation, the
scale amax/7, round-half-to-even, the [-7, 7] clamp, the fp32 rank-one
epilogue) the oracle follows the layer's written specification, and every
such reading is listed in the design notes.

Parity pins: every function here is pinned by a CPU test in
``tests/test_oracle_pins.py`` against something other than itself (library
routines, closed forms, brute force, hand-derived fixtures).  No function is
unpinned.
"""

from .w4a4_oracle import (  # noqa: F401
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    sylvester_hadamard,
    rotate_rows,
    gelu_f32,
    quantize_rows,
    pack_int4,
    unpack_int4,
    quantize_weight,
    quantize_activation,
    gemm_s32,
    epilogue,
    linear,
    boundary_window,
    lora_delta,
    linear_lora,
    requant_partials,
    chain_requant,
)
