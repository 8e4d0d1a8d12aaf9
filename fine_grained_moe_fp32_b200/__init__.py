"""dots.llm1 fine-grained MoE FFN layer on B200 (sm_100a).

The compute path lives in a C-ABI CUDA library (``libmoe_b200.so``, built from
``csrc/``); ``moe.py`` is a thin ctypes binding over it.  Importing the package
does not load the library; the first call does, and raises if it is missing.
"""
from .workloads import CONFIGS, MoEConfig, make_inputs  # noqa: F401
