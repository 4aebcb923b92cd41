"""B200-native Particle-Transformer pair-bias attention (sm_100a).

The CUDA library and its Python binding are loaded lazily by ``ops``; the
``synth`` and ``configs`` modules build seeded synthetic inputs.
"""
