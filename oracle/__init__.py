"""CPU oracle for the phase-specialised quantized linear layers.

TEST INFRASTRUCTURE ONLY: a plain, slow, obviously correct float64 / exact
restatement of what the GPU path computes.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import it.  The product path (the ``libnvq`` C-ABI library and
its Python binding) never imports, links or executes anything in here, and this
package imports nothing from the product path.

Modules:
  nvfp4     -- NVFP4 RTN quantization, dequantization, float64 GEMM reference,
               block-scale layout map (Mix-Quant page, section 2).
  int4      -- INT4 group-128 RTN quantization, W4A16 reference, the offline
               reorder and its inverse (MARLIN page).
  tiny_ref  -- independent pure-Python (Fraction) restatement for tiny inputs.
  swiglu    -- gate_up GEMM + SiLU * mul + NVFP4 with a static tensor scale,
               and the error-band comparison for its codes.
  sparse24  -- 2:4 magnitude pruning + INT4 group-128, the sparse W4A16
               reference, and the decode kernel's packed order with its inverse.

Every function here is pinned by CPU tests against values fixed by the pages
and by mathematics (closed forms, exhaustive brute force, hand-worked
examples); none is marked "parity unpinned".
"""
