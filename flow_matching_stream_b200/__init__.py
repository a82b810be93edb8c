"""Krea 2 single-stream MMDiT block and backbone forward on NVIDIA B200 (sm_100a).

The compute lives in ``libkrea2.so`` (hand-written CUDA behind the C ABI of
``include/krea2.h``); this package only marshals torch tensors into that ABI.
"""
from .krea2 import *  # noqa: F401,F403
