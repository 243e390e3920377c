"""CPU fp64 oracle for TurboQuant packed-KV quantize-append and paged decode.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the
``kv_cache_vector_append_b200`` package and its CUDA library) may import,
call, link or execute this package.  Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` use it.

The oracle is a plain, slow, obviously correct restatement of what the method
computes, written in numpy float64 from the pages that describe TurboQuant KV
compression.  It shares no code with the CUDA path.  See ``tq_oracle`` for the
functions and the passage each one follows, and ``gen_codebooks`` for the
script that writes the Lloyd-Max tables that both paths consume.

Parity status of each function (what pins it is listed in its docstring):
every function is pinned by a test under ``tests/test_oracle_*.py``; the
arbitrary conventions the pages leave open (sign generator, bit order inside a
byte, tie-break, GQA grouping) are pinned only by internal consistency and by
the published definitions they follow.
"""
