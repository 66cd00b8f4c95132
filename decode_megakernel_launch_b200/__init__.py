"""B200-native batch-1 Llama decode megakernel (W8A16): C-ABI library `libamk.so` plus a thin binding.

Importing the package does not load the CUDA library; `decode_megakernel_launch_b200.amk` does, and
raises if it is missing.
"""
__version__ = "0.1.0"
