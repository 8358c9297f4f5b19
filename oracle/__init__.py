"""CPU oracle for the GPT-2 training step -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this package. It shares no code with the CUDA path (gpt_step_b200/csrc) and
never calls it.
"""
from . import gpt2, philox  # noqa: F401
