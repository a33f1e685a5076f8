"""FAVOR+ attention hot path for NVIDIA B200 (sm_100a).

The work runs in hand-written CUDA kernels behind the C-ABI library ``libfavor.so`` (declared in
``include/favor.h``); ``api`` is its thin ctypes binding. Importing the package loads nothing;
the library is opened on first use and a missing or unbuilt library raises an error (there is no
CPU fallback).
"""
