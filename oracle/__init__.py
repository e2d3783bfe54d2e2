"""CPU oracle of the GPT-2 training step.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference arm, never by the product path.  See gpt2_oracle.py.
"""
from .gpt2_oracle import *  # noqa: F401,F403
