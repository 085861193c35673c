"""fp64 CPU oracle for gpt-oss-style sink-augmented grouped-query attention.

TEST INFRASTRUCTURE. This package is the plain, slow, obviously-correct
definition that the CUDA library is checked against. Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it; the product path (``sink_augmented_gqa_b200``) never does, and the two
share no code. Inputs come from the seeded generators in
``sink_augmented_gqa_b200.workloads``, which hold no attention arithmetic.

Modules, each citing the passage it restates:

* ``bf16``      -- exact round-to-nearest-even of fp64 values to bfloat16.
* ``yarn``      -- YaRN / NTK-by-parts inverse frequencies, concentration and
                   the cos/sin tables (MoE-Xtend README, "ROPE + SCALING").
* ``rope``      -- half-split rotary rotation at the global position
                   ``offset + local_t`` (MoE-Xtend README, "DESIGN CONTRACTS").
* ``attention`` -- masked GQA scores, the per-head sink column, softmax, the
                   dropped sink and the PV mix (MoE-Xtend README, "ATTENTION
                   STACK"; GQA Attention study note, "How it works").
* ``kvcache``   -- the append-only KV cache with snapshot / restore and the
                   KV-byte estimator (MoE-Xtend README, "KV CACHE").
* ``linear``    -- pre-norm RMSNorm, the fused qkv linear and the out
                   projection with the residual add (GQA Attention study
                   note, "How it works"; pinned by
                   ``tests/test_oracle_linear.py``).
* ``backward``  -- gradients of the attention with respect to q, k, v and
                   the sinks (GPT-OSS-Lite README: learned sinks, trained
                   end to end); pinned to finite differences by
                   ``tests/test_oracle_backward.py``.
* ``fp8``       -- E4M3 rows with one fp32 scale per row: quantise and
                   dequantise (MoE-Xtend README, "ROADMAP": KV quantisation
                   with dequantisation; the format is a reading, pinned by
                   ``tests/test_oracle_fp8.py``).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
except the two readings listed there as "parity unpinned" (the RoPE pair
convention against a real checkpoint, and the GPT-OSS-Lite rotary base).
"""

from . import bf16, yarn, rope, attention, kvcache, fp8, linear, backward  # noqa: F401
