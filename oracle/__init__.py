"""CPU oracle for MLA decoding over a paged KV cache (fp64, numpy).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The CUDA path
never calls into it, and it shares no code with the CUDA path: the two meet
only at the seeded inputs of ``mla_decode_attention_get_b200.inputs``.

Modules
-------
formats       bf16 / e4m3 / FP8-cache-row decoding, written from the format
              definitions.
mla_oracle    softmax(q K^T * scale) V and the log-sum-exp, walking the
              block_table; dense and sparse (top-k indices) key sets.
brute         the same definition as pure-Python loops, for tiny inputs.
metadata_ref  the split-KV scheduling plan, restated sequentially.
fp8_writer_ref  quantisation of new key rows into the FP8 cache row format
              (per-128 scale = max|x| / 448, e4m3 round-to-nearest-even).

Parity pins: every function here is pinned by ``tests/test_oracle_*.py``
against brute force, closed forms and invariants (no function is unpinned).
"""
