"""CPU oracles of the estimate -> select -> exact-attention path (prefill: ``prism_oracle``;
decode: ``fasa_oracle``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``, never by the library or its binding.
"""
