// Decode / probe kernels for 4-bit codes (one translation unit per pair, built in parallel).
#include "dwkv_decode.cuh"

DWKV_DECODE_INSTANTIATE(4, false)
