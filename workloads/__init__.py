"""Seeded synthetic workloads of the MoE expert layer: the input recipe that
both the CUDA path (tests, bench) and the CPU oracle consume.  It is neither
part of the library nor of the oracle."""
