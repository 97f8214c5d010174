// Decode / probe kernels for 4-bit codes, bf16 coefficients (one translation unit per triple, built in parallel).
#include "dwkv_decode.cuh"

DWKV_DECODE_INSTANTIATE(4, false, false)
