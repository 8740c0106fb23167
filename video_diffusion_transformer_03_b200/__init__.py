"""B200 (sm_100a) DiT-block denoising path behind the libh3b C ABI.

Submodules: ``h3b`` (ctypes binding; importing it requires the built libh3b.so),
``pipeline`` (device-resident synthetic denoiser), ``synth`` (seeded inputs) and
``build`` (nvcc build of the library).  Nothing is imported eagerly.
"""
__all__ = ["h3b", "pipeline", "synth", "build"]
