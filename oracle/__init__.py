"""CPU oracle (test infrastructure only).

Imported by the tests, by ``__graft_entry__.smoke()`` and by the CPU-baseline leg of
``bench.py`` -- never by the library or its binding. See ``fp4kv_oracle`` for the
definitions and the passages they follow.
"""
from .fp4kv_oracle import *  # noqa: F401,F403
