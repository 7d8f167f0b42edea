"""CPU oracle for the TurboQuant-prod / QJL compressed KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` (plus its ``--impl reference`` arm) may import or run it.  It
shares no code, table or constant generator with the CUDA library; the two
meet only in the seeded inputs of ``synth``.

Plain NumPy, float64 unless a step's storage precision is fixed (fp32 codebook,
projections and value metadata), no blocking, fusion or reordering.  Sources:

* [TQ]   TurboQuant KV-cache quantization article (kwkr.cn/news/562855):
         §二 three-stage pipeline, §四 QJL unbiasedness, §五 two-stage
         estimator, §六 attention scoring, store and ring buffer, §七 value
         quantization and known limits.
* [AQJL] A-QJL adaptive layer-wise KV compression article
         (zingnex.cn/forum/thread/a-qjl-kv): §QJL, §A-QJL, §实际部署 config.

Modules: ``philox`` (counter-based generator), ``projections`` (Pi, S),
``codebook`` (Lloyd-Max), ``quantize`` (keys, values), ``layout`` (packed
byte format), ``attention`` (logits, decode, chunk prefill), ``cache`` (append + ring),
``sensitivity`` (A-QJL layer groups and sketch dims from key variance).

Every function here is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_*.py``; no function is "parity unpinned".
"""
