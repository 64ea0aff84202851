"""Seeded synthetic prefill inputs shared by the oracle tests, the CUDA parity tests and the
benchmark.  Holds no part of the attention method itself."""
from .synthetic import (WORKLOADS, Workload, cu_seqlens_of, default_workers, dequantised,
                        generate)

__all__ = ["WORKLOADS", "Workload", "cu_seqlens_of", "default_workers", "dequantised", "generate"]
