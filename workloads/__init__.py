"""Seeded synthetic inputs for the multi-LoRA delta workloads.

This package only draws random numbers and lays out metadata (adapter ids,
segment offsets, request lists).  It holds none of the method's arithmetic:
no shrink, no expand, no routing.  Both the CUDA library's tests/benchmark and
the CPU oracle's tests take their inputs from here.
"""
from .configs import (  # noqa: F401
    Pool, BgmvCall, SgmvCall, MultiCall, Workload,
    make_pool, bgmv_call, sgmv_call, multi_call, zipf_ids,
    make_workload, WORKLOAD_NAMES, bf16_bits, to_host, cooccurrence_requests,
)
