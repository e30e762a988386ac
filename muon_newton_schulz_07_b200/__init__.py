"""Muon optimizer step for 2-D weight matrices on B200 (sm_100a).

The compute lives in the CUDA library ``libmuon.so`` (C ABI declared in
``include/muon.h``); ``binding`` marshals arguments to it and nothing more.
"""
