// Decode / probe kernels for 8-bit codes, probe variant, bf16 coefficients (one translation unit per triple, built in parallel).
#include "dwkv_decode.cuh"

DWKV_DECODE_INSTANTIATE(8, true, false)
