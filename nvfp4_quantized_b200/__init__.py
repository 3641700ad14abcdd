"""qt2: the Quartet II NVFP4 linear layer for B200 (sm_100a).

The compute path is the CUDA library ``libqt2.so`` behind the C ABI in ``include/qt2.h``;
``nvfp4_quantized_b200.qt2`` is its thin ctypes binding (argument marshalling only).
``nvfp4_quantized_b200.synth`` draws the seeded synthetic inputs.
"""
__all__ = ["qt2", "synth"]
