"""fp64 CPU oracle for MLA decode over a paged latent+RoPE cache.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it. The
library (``mla_latent_kv_46_b200``) never imports it and shares no code with it;
the only thing both sides use is the seeded input generator
(``inputs.workloads``), which holds no attention arithmetic and imports only numpy.

Sources (page title, then the section used):
  [GatedMLA]  kimi-k3 docs, "GatedMLA" (attention/gated_mla): "Projection geometry
              and stored weights", "Build per-head Q, K and V", "Observe logits,
              then compute causal attention", "Output projection and optional gate".
  [Primer]    modeldna.ai, "learn/mla": "Under the hood" and its cache-size table.
  [Ticket]    "MLA + KV cache (Tier 3 #5)": "Description", "Acceptance criteria".
  [Softved]   softved.com.np, "Introduction to MLA vs. KV Cache in Large Language
              Models": "Practical Implementation Tips for MLA in LLM Serving".
  [Tutorial]  "ARCH-MLA. Multihead Latent Attention | MLA 与紧凑 KV 表示":
              "Step 4：实现 KV 表示账本" (the KV-state ledger and its tests).

Modules:
  mla_oracle  the non-absorbed definition (reference semantics), the absorbed form,
              the split-KV log-sum-exp merge, cache append, full causal forward.
  loops       a scalar pure-Python restatement for tiny brute-force cases.
  ledger      the per-token KV-state byte ledger.
  fp8         the 8-bit (E4M3) cache: rounding, codes, per-token power-of-two scales.

Every function here is pinned by a ``-m "not gpu"`` test in tests/test_oracle.py
against something other than itself (closed forms, a library routine, brute force,
the pages' printed values). Nothing is "parity unpinned".
"""
