"""The CPU oracle for the NVFP4 MoE FFN layer.

TEST INFRASTRUCTURE.  This package is a plain, slow, fp64 restatement of what
the layer computes, written before and independently of the CUDA path: it
shares no code, headers, tables or helpers with ``moe_expert_layer_renorm_b200``
and never imports it (and vice versa).  Only ``tests/``, ``__graft_entry__``
(build and smoke) and ``bench.py``'s CPU-baseline and reference legs may
import it.

Two implementations of the same steps and readings, written apart:
  moe_oracle.cpp - plain C++ (fp64; fp32 where the format fixes it), the
                   oracle the GPU parity tests, the smoke check and the bench's
                   CPU legs use; also MXFP4 pack and decode (OCP MX v1.0) for
                   the MXFP4 expert variant; cpp.py is its ctypes front end,
                   build.py compiles it with g++
  nvfp4          - numpy: E2M1/E4M3 decode from bits, NVFP4 decode and pack
  moe_layer      - numpy: route, permute, SwiGLU expert FFN, combine, tolerance
  mxfp4          - numpy: MXFP4 (OCP MX) pack and decode, written apart from
                   the C++ one

Every function is pinned by a ``-m "not gpu"`` test against something other
than itself (hand-worked tables, closed forms, brute force, a library routine
for a special case); nothing is "parity unpinned".
"""
from . import nvfp4, moe_layer  # noqa: F401  (cpp is imported on demand: it compiles on first use)
