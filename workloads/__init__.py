"""Seeded synthetic workloads shared by the CUDA library's tests/bench and the CPU oracle."""
from .gen import (Data, Workload, WORKLOADS, SWEEP_BATCHES, generate, small, to_numpy,
                  splitmix64, bloom_bits, bloom_words)

__all__ = ["Data", "Workload", "WORKLOADS", "SWEEP_BATCHES", "generate", "small", "to_numpy",
           "splitmix64", "bloom_bits", "bloom_words"]
