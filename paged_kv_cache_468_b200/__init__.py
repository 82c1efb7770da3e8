"""B200-native paged KV-cache decode: the Python face of ``libpagedkv.so``.

Importing the package loads nothing; the CUDA library is opened on the first
call that needs it and a missing or unloadable library raises at that point.
There is no CPU fallback.
"""
