"""FAVOR attention oracle (plain fp64 CPU). Test infrastructure only.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline and reference legs may
import this package. The CUDA path shares no code with it.
"""
from .favor_oracle import *  # noqa: F401,F403
from .favor_oracle import TRIG, RELU  # noqa: F401
