// wd_testing.cu — entry points that exist only to test pieces of the
// kernels that no output of the path exposes on its own:
//   wd_test_exp2          the FMA-pipe 2^x of the attention softmax (and the
//                         MUFU ex2 beside it) evaluated on caller data;
//   wd_test_gelu          the GEMM epilogue's GELU (and the erff form of the
//                         CUDA-core path) evaluated on caller data;
//   wd_test_wait_timeout  one bounded mbarrier wait that nothing completes,
//                         with a short limit, so the timeout path (error
//                         word, drain, return, wd_check) can be exercised
//                         without any real pipeline stalling.
#include "wd_internal.cuh"

namespace wd {

__global__ void k_test_exp2(const float* __restrict__ x, float* __restrict__ y_fma, float* __restrict__ y_fma2,
                            float* __restrict__ y_mufu, float* __restrict__ y_lib, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = x[i];
    y_fma[i] = tca::exp2_fma(v);
    // the packed form on the pair (x[i], x[i ^ 1]): lane 0 is x[i]
    const int64_t j = ((i ^ 1) < n) ? (i ^ 1) : i;   // the partner index, inside [0, n)
    y_fma2[i] = tca::exp2_fma2(make_float2(v, x[j])).x;
    y_mufu[i] = tca::ex2(v);
    y_lib[i] = exp2f(v);
  }
}

__global__ void k_test_gelu(const float* __restrict__ x, float* __restrict__ y_as, float* __restrict__ y_as2,
                            float* __restrict__ y_erf, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    y_as[i] = gelu_as(x[i]);
    // the packed form on the pair (x[i], x[i ^ 1]): lane 0 is x[i]
    const int64_t j = ((i ^ 1) < n) ? (i ^ 1) : i;
    y_as2[i] = gelu_as2(make_float2(x[i], x[j])).x;
    y_erf[i] = gelu_erf(x[i]);
  }
}

// One warp waits (as a whole warp, like the softmax warps) on phase 0 of an
// mbarrier with one expected arrival that never comes.  The wait gives up
// after limit_ns, records `site` in the device error word and the kernel
// returns; out[0] = 1 if the wait reported completion, 0 if it ran out.
__global__ void k_test_wait_timeout(uint64_t limit_ns, unsigned site, int* out) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const bool ok = __all_sync(0xffffffffu, mbar_wait_limit(&bar, 0u, site, limit_ns));
  if (threadIdx.x == 0) out[0] = ok ? 1 : 0;
}

}  // namespace wd

extern "C" {

wd_status wd_test_exp2(const float* x, float* y_fma, float* y_fma2, float* y_mufu, float* y_lib, int64_t n,
                       wd_stream stream) {
  using namespace wd;
  WD_NEED(x); WD_NEED(y_fma); WD_NEED(y_fma2); WD_NEED(y_mufu); WD_NEED(y_lib);
  if (n <= 0) { set_error("wd_test_exp2: n = %lld", (long long)n); return WD_ERR_SHAPE; }
  const int64_t blocks = (n + 255) / 256;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Trace tr(KC_SMALL, st);
  k_test_exp2<<<static_cast<unsigned>(blocks < 4096 ? blocks : 4096), 256, 0, st>>>(x, y_fma, y_fma2, y_mufu, y_lib, n);
  return launch_status("test_exp2");
}

wd_status wd_test_gelu(const float* x, float* y_as, float* y_as2, float* y_erf, int64_t n, wd_stream stream) {
  using namespace wd;
  WD_NEED(x); WD_NEED(y_as); WD_NEED(y_as2); WD_NEED(y_erf);
  if (n <= 0) { set_error("wd_test_gelu: n = %lld", (long long)n); return WD_ERR_SHAPE; }
  const int64_t blocks = (n + 255) / 256;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Trace tr(KC_SMALL, st);
  k_test_gelu<<<static_cast<unsigned>(blocks < 4096 ? blocks : 4096), 256, 0, st>>>(x, y_as, y_as2, y_erf, n);
  return launch_status("test_gelu");
}

wd_status wd_test_wait_timeout(uint64_t limit_ns, unsigned site, int* out, wd_stream stream) {
  using namespace wd;
  WD_NEED(out);
  if (limit_ns == 0 || limit_ns > 100000000ull) {
    set_error("wd_test_wait_timeout: limit %llu ns outside (0, 100 ms]", (unsigned long long)limit_ns);
    return WD_ERR_ARG;
  }
  if (site == 0) { set_error("wd_test_wait_timeout: site 0 is reserved for 'no error'"); return WD_ERR_ARG; }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Trace tr(KC_SMALL, st);
  k_test_wait_timeout<<<1, 32, 0, st>>>(limit_ns, site, out);
  return launch_status("test_wait_timeout");
}

}  // extern "C"
