"""Seeded synthetic inputs for the lightning-indexer selection path.

This package is shared by the oracle, the tests and the benchmark.  It only
draws random numbers and stores them in the byte formats the indexer reads
(bf16, fp8 e4m3 with a per-key fp32 scale, int8 with a per-key fp32 scale, PQ
codes with fp16 codebooks trained by k-means on the keys); it holds none of the
scoring or selection arithmetic.
"""

from .shapes import WORKLOADS, Workload, get_workload  # noqa: F401
from .synth import (  # noqa: F401
    make_decode,
    make_prefill,
    make_two_stage,
    make_bucket,
    make_workload,
)
