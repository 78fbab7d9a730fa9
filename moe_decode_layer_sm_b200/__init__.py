"""B200-native fused decode FFN half-layer ("mono" kernel): a C-ABI CUDA
library (libmonoffn.so, include/mono_ffn.h) and its thin Python binding."""

from .binding import Plan, MonoError, lib  # noqa: F401
