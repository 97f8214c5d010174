// Decode / probe kernels for 8-bit codes (one translation unit per pair, built in parallel).
#include "dwkv_decode.cuh"

DWKV_DECODE_INSTANTIATE(8, false)
