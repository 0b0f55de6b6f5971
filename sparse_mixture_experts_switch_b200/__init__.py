"""Switch-FFN layer forward pass for one NVIDIA B200 (sm_100a).

The work happens in libswitchmoe.so (C ABI: include/switch_moe.h);
``switch_moe`` is its Python binding.
"""
