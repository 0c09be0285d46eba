"""fp64 CPU oracle of the Qwen3 decoder block -- test infrastructure only.

Imported by tests/, __graft_entry__.smoke() and the CPU-baseline leg of bench.py;
never by the CUDA library or its Python binding. qwen3_ref.py states the definitions
in numpy (with the citations); qwen3_ref.cpp states them again in plain C++ loops,
reached through cpp_ref.py with the same function signatures, and both answer to the
same pins.
"""
from .qwen3_ref import *  # noqa: F401,F403
from . import qwen3_ref  # noqa: F401
