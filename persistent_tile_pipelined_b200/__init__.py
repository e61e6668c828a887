"""Persistent tile engine for batch-1 LLM decode on B200 (sm_100a).

The engine itself is ``libtre.so`` (C ABI declared in ``include/tre.h``); the Python
binding in ``tre.py`` only marshals arguments.  Import ``persistent_tile_pipelined_b200.tre``
for the engine; it raises if the native library is missing.
"""
