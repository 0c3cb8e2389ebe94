"""CPU oracle for the fused MoE expert layer: TEST INFRASTRUCTURE ONLY.

This package is the slow, plain, float64 statement of what the MoE expert layer
computes.  It exists so that the CUDA path can be checked against something that a
reader can compare with the source pages by eye.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import it.  The product path (the C-ABI library and its Python
binding) never imports, links or executes anything in here, and this package
imports nothing from the product package.

Sources (web pages, cited by title and section):
  [SwiGLU PR]   DeepGEMM PR #445 "fix(sm90): support parameterized SwiGLU in FP8
                MegaMoE" -- Summary (OAI-SwiGLU formula), Root Cause, Compatibility
                (defaults alpha=1, up_bias=0).
  [SM100 PR]    DeepGEMM PR #386 "Optimize sm100 version with token-aware BM240
                tiling, native UE8M0, and direct combine" -- title and Description.
  [o_proj PR]   TensorRT-LLM PR #16346 "DSV4 o_proj: fuse fp8/UE8M0 quantize ..." --
                Description (fused BF16->FP8 + 1x128 UE8M0 quantisation, amax).
  [sched PR]    fw-ai/DeepGEMM PR #16 "Sync upstream through PR #441: fix Mega MoE
                scheduler ordering" -- Overview.
The element formats (E4M3, E2M1, UE8M0) are the OCP Microscaling / FP8 formats
the pages name but do not define; their definitions are written out in
``formats.py``.

Parity status per function is stated in each module's header.
"""
