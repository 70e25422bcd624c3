"""Plain, slow CPU oracle for the W4A4 NVFP4 linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.
It shares no code with the CUDA path (``bit_diffusion_transformer_nvfp4_b200``)
and never imports it.

Modules
-------
``nvfp4``   the NVFP4 number formats (E2M1 element codes, E4M3 block scales,
            FP32 per-tensor scale) and the tensor quantiser, in IEEE fp32 where
            the quantiser takes a rounding decision, fp64 everywhere else.
``linear``  the dual-branch W4A4 forward pass in fp64.
``prep``    offline SVDQuant preparation: smoothing factors, truncated SVD,
            low-rank factors and the residual weight.
``gelu``    the tanh-approximated GELU in fp64.
"""
