// common.cuh -- small device/host helpers shared by the library's kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "../../include/mla.h"

namespace mla {

// ---------------------------------------------------------------------------------------------
// element conversion
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(__nv_fp8_e4m3 x) { return static_cast<float>(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
// e4m3: round to nearest even, saturating to +-448 (the format has no infinity)
template <> __device__ __forceinline__ __nv_fp8_e4m3 from_f32<__nv_fp8_e4m3>(float x) {
  __nv_fp8_e4m3 r;
  r.__x = __nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
  return r;
}

// ---------------------------------------------------------------------------------------------
// device status word: set by bounded waits that gave up; read and cleared by mla_check_status
// ---------------------------------------------------------------------------------------------
// Kernels with bounded waits receive the word's device address and the spin limit as parameters.
int* device_status_ptr();        // device address of the status word on the current device
long long wait_limit();          // nanoseconds before a bounded device wait gives up
void set_wait_limit(long long);  // 0 restores the default

__device__ __forceinline__ void report_timeout(int* status) {
  if (status) atomicExch(status, (int)MLA_ERR_TIMEOUT);
}

// ---------------------------------------------------------------------------------------------
// host helpers
// ---------------------------------------------------------------------------------------------
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t round_up(size_t a, size_t b) { return (a + b - 1) / b * b; }
inline size_t dtype_bytes(int32_t dt) { return dt == MLA_BF16 ? 2 : (dt == MLA_FP8_E4M3 ? 1 : 4); }

int sm_count();          // multiprocessors of the current device (cached per device)
int current_device();

void count_launch();      // one more kernel launched by this library (see mla_launch_count)
long long launch_count();

// Programmatic dependent launch. The hot-path kernels are launched with launch_pdl: such a kernel may
// begin (prologue: barriers, tensor memory, descriptor prefetch) while the previous kernel of the
// stream is still running. Every CTA calls griddep_wait() before it touches memory that earlier work
// in the stream writes or reads; it returns once the previous kernel has completed and its writes are
// visible (a no-op without a programmatic dependency). Because every such kernel waits in every CTA,
// completion stays ordered through the whole chain. griddep_launch_dependents() lets the next kernel
// start launching once every CTA of this grid has called it or exited (all CTAs are then resident,
// so the early start cannot take SMs that this grid still needs).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

void count_launch();

template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  count_launch();
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

// after every kernel launch: count it and turn a launch error into MLA_ERR_CUDA
#define MLA_LAUNCH_CHECK()                                   \
  do {                                                       \
    ::mla::count_launch();                                   \
    if (cudaPeekAtLastError() != cudaSuccess) {              \
      (void)cudaGetLastError();                              \
      return MLA_ERR_CUDA;                                   \
    }                                                        \
  } while (0)

// ---------------------------------------------------------------------------------------------
// CUDA-core kernels (any dims; fp32 accumulate). Launchers return an mla status.
// ---------------------------------------------------------------------------------------------
struct GemmArgs {
  // C[b][m][n] = epi( sum_k A[b][m][k] * B[b](n, k) ) (* G[b][m][n] when G != nullptr)
  const void* A; int64_t sa_b, sa_m, sa_k;
  const void* B; int64_t sb_b, sb_n, sb_k;
  void* C;       int64_t sc_b, sc_m, sc_n;
  const void* G; int64_t sg_b, sg_m, sg_n;
  int64_t M, N, K, batch;
  int sigmoid;
};

// a_dt / b_dt / c_dt / g_dt: MLA_F32 or MLA_BF16 for each operand
int gemm_generic(const GemmArgs& args, int32_t a_dt, int32_t b_dt, int32_t c_dt, int32_t g_dt,
                 cudaStream_t stream);

int copy_rows_strided(const void* src, int64_t src_stride, void* dst, int64_t dst_stride,
                      int64_t rows, int64_t cols, int32_t dt, cudaStream_t stream);

int append_latent_launch(const mla_dims& d, int32_t cache_dtype, void* cache, int64_t cache_rows,
                         const int64_t* row_idx, const float* c_new, const float* kpe_new,
                         const int32_t* positions, int64_t n_new, uint32_t flags, float eps,
                         float theta, cudaStream_t stream);

// the same with row strides (in floats) of c_new and kpe_new
int append_latent_strided(const mla_dims& d, int32_t cache_dtype, void* cache, int64_t cache_rows,
                          const int64_t* row_idx, const float* c_new, int64_t c_stride, const float* kpe_new,
                          int64_t kpe_stride, const int32_t* positions, int64_t n_new, uint32_t flags,
                          float eps, float theta, cudaStream_t stream, float cache_scale = 1.f);
// log-sum-exp merge of n_parts partial decode results (rows row0 .. row0 + n_rows of each part)
int lse_merge_launch(int n_parts, const float* const* o_parts, const float* const* l_parts, int64_t row0,
                     int64_t n_rows, int H, int dc, float* out_lat, float* lse, cudaStream_t stream);

// out[t, h, :] = R_{positions[t]} src[t, h, :] (rotate) or src[t, h, :]: src fp32 [n_rows, H, dr],
// out in dtype
int rope_rows_launch(int32_t dtype, const float* src, void* out, const int32_t* positions, int64_t n_rows, int H,
                     int dr, bool rotate, float theta, cudaStream_t stream, int n_parts = 1,
                     int64_t part_stride = 0);

struct DecodeArgs {
  const void* q_abs; const void* cache; const int32_t* cu_seqlens;
  int32_t batch, n_q, H, dc, dr; int64_t max_seqlen, total_rows;
  float scale; bool causal;
  float* out_lat; float* lse;
  void* workspace; size_t workspace_bytes;
  float cache_scale = 1.f;               // an e4m3 cache holds value / cache_scale
  bool cache_f8 = false;                 // the cache is e4m3 (tensor-core decode with a bf16 query)
  void* out_lat_bf16 = nullptr;          // tensor-core decode: write out_lat here in bf16 instead
};

size_t decode_generic_workspace(const DecodeArgs& a);
// dtype: of q_abs and the cache (MLA_F32 or MLA_BF16); cache_dtype MLA_FP8_E4M3 takes an e4m3 cache
// with a bf16 or fp32 query
int decode_generic_launch(const DecodeArgs& a, int32_t dtype, cudaStream_t stream, int32_t cache_dtype = -1);

}  // namespace mla
