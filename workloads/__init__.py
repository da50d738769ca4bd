"""Seeded synthetic inputs for the KDA recurrence workloads.

This package is shared by the CPU oracle's tests and the GPU path's tests and
benchmark.  It only draws random numbers and shapes them into the input
distributions each workload names; it holds none of the recurrence, prologue
or chunk arithmetic.
"""
from .kda_inputs import *  # noqa: F401,F403
