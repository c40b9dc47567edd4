"""Displaced-patch UNet layer step (DistriFusion's patch-parallel hot path) on one B200.

Submodules: ``configs`` (the named workloads), ``inputs`` (seeded synthetic
inputs), ``build`` (compiles csrc/ into libdfp.so), ``dfp`` (ctypes binding of
the C ABI in include/dfp.h; importing it requires the built library).
"""
