"""fp64 CPU oracle for sparse spatiotemporal video attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports, links or runs this
package.  Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
reference leg may call it.

It is a plain, slow restatement of what the hot path computes, written from
these pages:

* "Token Radius Attention for Efficient Video Generation" (gist.science
  summary): dense 3D softmax attention (1. Problem Statement), block-level
  sparsity, per-query entropy and a radius neighbourhood (2. Methodology:
  Insight I, Insight II, The TRA Pipeline, including its tile-major token
  layout).
* "Radial Attention to Accelerate Video Generation" (blog): a static mask
  whose window shrinks with frame distance (The idea behind Radial Attention).
* "Where Compute Matters: Heterogeneous Attention for Efficient Video
  Diffusion": uncertain tokens to dense global attention, the rest to local
  attention (Abstract).
* "AB-Attention speeds up video diffusion transformers up to 2.23x, no
  training" (Glonce): intra-block clustering selector (IBCS), sampling with
  inclusion-probability weighting (SIP) (method paragraph, Key facts).
* "DynamicRad: Content-Adaptive Sparse Attention for Long Video Diffusion":
  static-ratio and dynamic-threshold selection inside a radial prior
  (Abstract).

Floating point is fp64 unless a page fixes the precision; inputs are the
same bf16/fp32 values the library receives, widened exactly.  Library
primitives (numpy matmul, sort) serve as single steps; there is no tiling,
fusion or reordering beyond the definitions.

Parity status of each function is stated in its module docstring; every
function here is pinned by a `-m "not gpu"` test in tests/test_oracle_*.py
against closed forms, invariants, brute force on tiny grids or an
independent library routine.
"""
