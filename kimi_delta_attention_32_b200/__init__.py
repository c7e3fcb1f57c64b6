"""libkda: Kimi Delta Attention (KDA) on B200 (sm_100a).

The compute lives in ``libkda.so`` (CUDA kernels behind the C ABI declared in
``include/kda.h``); ``kda`` is its ctypes binding and ``workloads`` makes seeded
synthetic inputs. Importing the package does not load the library; the first
call does, and raises if the library is missing.
"""
from . import kda, workloads  # noqa: F401

__all__ = ["kda", "workloads"]
