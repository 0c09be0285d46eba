"""fp64 CPU oracle of the Qwen3 decoder block -- test infrastructure only.

Imported by tests/, __graft_entry__.smoke() and the CPU-baseline leg of bench.py;
never by the CUDA library or its Python binding. See qwen3_ref.py for the
definitions and the citations.
"""
from .qwen3_ref import *  # noqa: F401,F403
from . import qwen3_ref  # noqa: F401
