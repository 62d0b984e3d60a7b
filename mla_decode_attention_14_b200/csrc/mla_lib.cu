// mla_lib.cu -- single translation unit of the library (the device error word and all
// kernels live in one module, so no separate device linking is needed).
#include "api.cu"
#include "metadata.cu"
#include "combine.cu"
#include "decode_sm100.cu"
#include "noalloc.cu"
#include "selftest.cu"
#include "append.cu"
#include "head_gemm.cu"
