"""CPU oracle of the block-diffusion denoising step.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only `tests/`,
`__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py` may import
or run anything in this package.  The CUDA library never calls it, and it
shares no code, header, table or constant generator with the CUDA path; the
only module both sides use is `block_text_diffusion_b200.inputs` (seeded
random inputs, none of the method's arithmetic).

Modules:
  numerics -- Philox4x32-10, own binary32 log / exp / cos(2 pi u), bf16
              rounding (published definitions, fixed op sequences)
  sampler  -- entropy, temperature schedule, Gumbel-max sampling, commit /
              re-noise, adaptive stop
  model    -- weights, causal prompt encode, one denoising step, block loop

Parity status: every building block is pinned by tests/test_oracle_*.py
against closed forms, brute force or published test vectors, and the
composed model (prompt encode, canvas forward, denoising step, block loop)
against an element-by-element brute-force evaluation on a micro
configuration and against the method's invariants.  The pages print no
numeric worked example; what stays unpinned is only the bf16
double-rounding behaviour of the composed model at sizes beyond the micro
brute force (the bf16 storage points themselves are pinned by unit tests of
`store`).
"""
from . import numerics, sampler, model  # noqa: F401
