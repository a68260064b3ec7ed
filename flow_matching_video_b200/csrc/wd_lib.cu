// wd_lib.cu — libwd is built as one translation unit so that every kernel
// sees the same device error word without relocatable device code.
#include "wd_trace.cu"
#include "k_small.cu"
#include "k_simt.cu"
#include "k_gemm_tc.cu"
#include "k_attn_tc.cu"
#include "k_attn_f8.cu"
#include "wd_api.cu"
#include "wd_noalloc.cu"
#include "wd_testing.cu"
