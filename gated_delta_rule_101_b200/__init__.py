"""B200-native Kimi Delta Attention (KDA): a thin Python binding over libkda.

The binding is filled in alongside the CUDA library.
"""
