// Decode / probe kernels for 4-bit codes, coefficients in the 8-bit blockwise form (one
// translation unit per triple, built in parallel).
#include "dwkv_decode.cuh"

DWKV_DECODE_INSTANTIATE(4, false, true)
