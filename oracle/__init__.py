"""CPU oracle of the MoE expert layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never calls it and has no CPU fallback.

It is a plain, slow, obviously correct restatement, in numpy fp64, of what the
layer computes, written from the method's description:

* "Ai2 rebuilds Olmo's training stack for trillion-parameter MoEs"
  (alphasignal.ai) -- introduction (a router sends each token to a small
  selection of feed-forward experts), "Routing work stays on the GPU" (routed
  token rows written straight into expert input buffers; grouped GEMM over the
  experts), "MXFP8 reduces compute and memory costs" (8-bit floats with one
  scale per small block);
* "Supercharging Olmo-core for Efficient and Scalable MoE Training"
  (papers.projxon.ai) -- Summary (rowwise dispatch into expert buffers,
  GPU-resident routing metadata, device-scheduled grouped GEMMs, MXFP8).

The pages give no formula; the readings taken where they are silent (softmax
top-k with renormalisation, lowest-index tie-break, SwiGLU experts, ascending
token order inside an expert, OCP MX v1.0 block scaling) are stated in the
module and function docstrings.

Modules:
  numerics -- bf16 / fp32 rounding, OCP FP8 E4M3 and E8M0 block scaling
  moe      -- router, dispatch plan, expert FFN, combine, backward, MXFP8 GEMM
  ref_c    -- ctypes binding of ``moe_ref.c``: the whole layer again, in plain
              C99 fp64 loops per token and selected expert, with its own bf16
              rounding and E4M3 encoder (built by ``make`` in this directory)

Every function is pinned by ``tests/test_oracle_pins.py`` and
``tests/test_oracle_c.py`` to closed forms, invariants, library routines and
finite differences -- never to the GPU path -- and the two statements of the
layer are checked against each other.
"""
from . import numerics, moe  # noqa: F401
