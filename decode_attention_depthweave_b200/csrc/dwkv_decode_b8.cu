// Decode / probe kernels for 8-bit codes, bf16 coefficients (one translation unit per triple, built in parallel).
#include "dwkv_decode.cuh"

DWKV_DECODE_INSTANTIATE(8, false, false)
