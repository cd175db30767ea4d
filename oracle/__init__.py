"""CPU oracle for low-bit MLA decode -- TEST INFRASTRUCTURE, not product code.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline
leg and its ``--impl reference`` arm) may import anything from this package.
The library under ``bit_mla_kv_qdecode_b200`` never imports it and shares no
code with it; the only thing both sides consume is the seeded input generator
``bit_mla_kv_qdecode_b200.synth``, which holds none of the method's arithmetic.

What it computes, and where each piece comes from:

* ``quant``     -- per-token, per-group asymmetric round-to-nearest quantizer
                   (INT4 or INT2), bit packing and dequantization. The method
                   caches both MLA paths in low bit widths: joint INT4, or INT2
                   content with INT4 RoPE (QuantMLA, arxivdaily.com/papers/
                   2609.36760, English abstract). Its baselines use plain
                   round-to-nearest with "the same quantizer as QuantMLA"
                   (QuantMLA podcast episode, researchpod.app, the passage on
                   baselines). Group size, fp16 scale and zero-point are the
                   workload's parameters.
* ``layout``    -- the packed page layout (codes + metadata per 64-token page)
                   and the paged cache writer / reader.
* ``attention`` -- dequantize-then-attend in float64, in the absorbed MQA form
                   of MLA decode (Group-Query Latent Attention abstract,
                   thelatestinai.com/papers/2607.27269: trained MLA weights
                   expose one decoding path, an absorbed MQA form), plus the
                   split-KV log-sum-exp merge and the unquantized BF16 decode.

Every function is pinned by tests in ``tests/test_oracle_*.py`` against
something other than itself: closed forms, brute force on tiny inputs
(including explicit non-absorbed MLA with per-head up-projections),
invariants and hand-derived worked examples.
"""
