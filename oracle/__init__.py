"""Plain fp64 CPU oracle for single-step Multi-Head Latent Attention decode.

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline / ``--impl reference`` legs
of ``bench.py`` may import this package. The CUDA library and its Python
binding (``latent_kv_decode_b200``) never import it, and it imports nothing
from them: the two share no kernels, helpers, tables or constants. Inputs for
both come from ``latent_kv_decode_b200.workloads``, which only draws random
numbers and lays them out.

Everything is computed in float64 from the storage-dtype values of the inputs
(fp32 or bf16, upcast exactly). Library routines (``np.einsum``, ``np.exp``)
serve as steps; there is no blocking, fusion or reordering beyond what the
definitions state.

Modules:

- ``oracle.mla``: absorbed decode (``mla_decode_step`` of the 6547.cn "MLA
  单步解码" exam question, blanks [1]-[5]), the naive decompressed form it must
  equal, visibility (mask / ragged lengths / causal speculative tokens), the
  paged gather, and the split-KV partials with their log-sum-exp merge.
- ``oracle.v41``: the DeepSeek-V4.1-Flash shared-latent variant (openarchlab
  "4A · Multi-head Latent Attention"): E2M1/E4M3 decoding of the 288-byte FP4
  cache entry, the FP4 quantiser of the cache-write step, RoPE on the last 64
  latent dims and its inverse, and the decode with one sink logit per head.

Pins (``tests/test_oracle_*.py``, CPU only) tie each function to something
other than itself: the printed demo shape, the decompressed-MHA identity,
closed forms, invariants, exhaustive format tables checked against torch's
float8 conversion and the OCP E2M1 value set, and RoPE's complex-rotation
form. Which pin covers which function is listed in each module's docstring.
"""
