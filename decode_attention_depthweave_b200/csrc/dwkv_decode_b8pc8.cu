// Decode / probe kernels for 8-bit codes, probe variant, coefficients in the 8-bit blockwise form (one
// translation unit per triple, built in parallel).
#include "dwkv_decode.cuh"

DWKV_DECODE_INSTANTIATE(8, true, true)
