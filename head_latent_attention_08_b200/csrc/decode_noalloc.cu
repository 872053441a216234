// decode_noalloc.cu -- mla_decode_absorbed_noalloc: the absorbed decode with its scratch in a fixed
// device array of this library instead of a caller-provided workspace. It allocates nothing: the
// array is part of the module's device image, and its address is looked up once per device.
#include <mutex>

#include "common.cuh"

namespace {

// Scratch of the decode: the per-block tile prefix, then the split partials (two slots of
// 128 rows x 512 latent columns fp32 per 2-CTA cluster, at most 74 clusters on a 148-SM B200:
// 37 MiB) and their row maxima and sums. Nothing in it has to start at zero: the plan kernel writes
// the prefix and every partial slot is written before it is read, within each call.
constexpr size_t kScratchBytes = MLA_DECODE_NOALLOC_MAX_BYTES;
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the array on the current device (looked up once per device, with that device
// current); nullptr if the lookup fails.
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) {
      (void)cudaGetLastError();
      return nullptr;
    }
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" int32_t mla_decode_absorbed_noalloc(const mla_dims* dims, int32_t dtype, const void* q_abs,
                                               const void* cache, const int32_t* cu_seqlens, int32_t batch,
                                               int32_t n_q, int64_t max_seqlen, int64_t total_rows,
                                               uint32_t flags, float* out_lat, float* lse, void* stream) {
  size_t need = 0;
  int32_t st = mla_decode_workspace_size(dims, dtype, batch, n_q, max_seqlen, total_rows, flags, &need);
  if (st != MLA_OK) return st;
  if (need > kScratchBytes) return MLA_ERR_WORKSPACE;
  // the scratch address is the current device's: a stream of another device would hand its kernels
  // an address that is not theirs, so such a call is refused before any launch
  int cur = -1, sdev = -1;
  if (cudaGetDevice(&cur) != cudaSuccess ||
      cudaStreamGetDevice(reinterpret_cast<cudaStream_t>(stream), &sdev) != cudaSuccess) {
    (void)cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  if (sdev != cur) return MLA_ERR_CUDA;
  void* scratch = scratch_on_current_device();
  if (!scratch) return MLA_ERR_CUDA;
  return mla_decode_absorbed(dims, dtype, q_abs, cache, cu_seqlens, batch, n_q, max_seqlen, total_rows, flags,
                             out_lat, lse, scratch, kScratchBytes, stream);
}
