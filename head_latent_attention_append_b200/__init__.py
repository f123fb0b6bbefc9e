"""B200-native multi-head latent attention on a paged latent cache.

Submodules: ``mla`` (ctypes binding over libmla's C ABI; importing it fails if
libmla.so is not built), ``synth`` (seeded synthetic inputs), ``workload``
(device-resident workload setup), ``build`` (nvcc build of libmla.so).
"""
