// wd_noalloc.cu — patch embedding for callers that cannot allocate device
// memory: the scratch of the patch gather lives in a fixed device array of
// this library instead of a caller-provided workspace.
#include <mutex>

#include "wd_internal.cuh"

namespace wd {

// The scratch holds the gathered patches, [batch * L, K] in the storage type
// (K = 144 for the image-to-video model, 64 for the text-to-video model).
// Every device that loads this library reserves it until the process exits.
static __device__ __align__(256) unsigned char g_patch_scratch[WD_NOALLOC_PATCH_SCRATCH_BYTES];

// Device address of the scratch on the current device, looked up once per
// device (the name alone is a host-side stand-in, not a device address).
static wd_status patch_scratch(void** out) {
  static std::mutex mu;
  static void* ptr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) {
    set_error("wd_patch_embed_noalloc: no usable current device (%s)", cudaGetErrorString(e));
    return WD_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_patch_scratch);
    if (e != cudaSuccess || p == nullptr) {
      set_error("wd_patch_embed_noalloc: cudaGetSymbolAddress failed (%s)", cudaGetErrorString(e));
      return WD_ERR_CUDA;
    }
    ptr[dev] = p;
  }
  *out = ptr[dev];
  return WD_OK;
}

}  // namespace wd

extern "C" wd_status wd_patch_embed_noalloc(const wd_dims* d, const float* x_t, const float* y, const void* w,
                                            const float* b, int batch, float* X, wd_stream stream) {
  using namespace wd;
  WD_TRY(check_dims(d));
  WD_TRY(check_batch(batch));
  WD_NEED(x_t); WD_NEED(w); WD_NEED(b); WD_NEED(X);
  if (d->n_img > 0) { WD_NEED(y); } else { WD_OPT(y); }
  const int64_t rows = batch * tokens(d);
  const int K = patch_k(d);
  const size_t need = static_cast<size_t>(rows) * K * esize(d);
  if (need > WD_NOALLOC_PATCH_SCRATCH_BYTES) {
    set_error("wd_patch_embed_noalloc: %lld token rows need %zu bytes of scratch, more than the fixed %u "
              "(at most %zu rows); use wd_patch_embed with a workspace", (long long)rows, need,
              WD_NOALLOC_PATCH_SCRATCH_BYTES, static_cast<size_t>(WD_NOALLOC_PATCH_SCRATCH_BYTES) / (K * esize(d)));
    return WD_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  WD_TRY(patch_scratch(&scratch));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t n = rows * K;   // every scratch element is written below: nothing to clear
  const unsigned grid = static_cast<unsigned>((n + 255) / 256 < 65536 ? (n + 255) / 256 : 65536);
  if (d->dtype == WD_BF16) {
    { Trace tr(KC_SMALL, st); k_patch_gather<bf16><<<grid, 256, 0, st>>>(x_t, y, batch, d->T, d->H, d->W, K, static_cast<bf16*>(scratch)); }
    WD_TRY(launch_status("patch_gather"));
    WD_TRY(gemm<bf16>(static_cast<int>(rows), d->D, K, scratch, K, w, K, EPI_F32, epi(X, d->D, b), st));
  } else {
    { Trace tr(KC_SMALL, st); k_patch_gather<float><<<grid, 256, 0, st>>>(x_t, y, batch, d->T, d->H, d->W, K, static_cast<float*>(scratch)); }
    WD_TRY(launch_status("patch_gather"));
    WD_TRY(gemm<float>(static_cast<int>(rows), d->D, K, scratch, K, w, K, EPI_F32, epi(X, d->D, b), st));
  }
  return WD_OK;
}
