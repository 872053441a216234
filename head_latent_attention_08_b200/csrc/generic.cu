// generic.cu -- CUDA-core kernels of the library: any dims, fp32 or bf16 storage, fp32 arithmetic.
//
// These carry the fp32 workloads (where tensor-core tf32 would not meet a 1e-4 tolerance) and
// every shape the tensor-core kernels do not take:
//   * gemm_generic: a strided, batched C = A . B^T with fp32 accumulation (query absorption,
//     weight folding, value/output projection, dense linear);
//   * append_latent_kernel: the latent-cache append with optional RMSNorm and RoPE;
//   * decode_generic_kernel + decode_combine_kernel: split-KV absorbed decode with an online
//     softmax held per head by one warp (shuffle max/sum), and the log-sum-exp merge of splits.
#include <math.h>
#include <string.h>

#include <atomic>

#include "common.cuh"

namespace mla {

// device status word (one per device that loads the library)
static __device__ int g_device_status = 0;
static long long g_wait_limit_host = 0;
constexpr long long kDefaultWaitLimit = 2000000000LL;  // 2 s of the device's global timer

int* device_status_ptr() {
  static int* cached[64] = {nullptr};
  const int d = current_device();
  if (d < 0 || d >= 64) return nullptr;
  if (!cached[d]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) {
      (void)cudaGetLastError();
      return nullptr;
    }
    cached[d] = static_cast<int*>(p);
  }
  return cached[d];
}

static std::atomic<long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
long long launch_count() { return g_launches.load(std::memory_order_relaxed); }

long long wait_limit() { return g_wait_limit_host > 0 ? g_wait_limit_host : kDefaultWaitLimit; }
void set_wait_limit(long long v) { g_wait_limit_host = v > 0 ? v : 0; }

int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

int sm_count() {
  static int cached[64] = {0};
  int d = current_device();
  if (d < 0 || d >= 64) return 148;
  if (cached[d] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0) n = 148;
    cached[d] = n;
  }
  return cached[d];
}

// ---------------------------------------------------------------------------------------------
// strided batched GEMM, 64 x 64 tile, 256 threads, 4 x 4 outputs per thread
// ---------------------------------------------------------------------------------------------
template <typename TA, typename TB, typename TC, typename TG>
__global__ void __launch_bounds__(256) gemm_generic_kernel(GemmArgs a) {
  __shared__ float As[16][68];
  __shared__ float Bs[16][68];
  const int64_t bz = blockIdx.z;
  const int64_t m0 = (int64_t)blockIdx.y * 64, n0 = (int64_t)blockIdx.x * 64;
  const TA* A = static_cast<const TA*>(a.A) + bz * a.sa_b;
  const TB* B = static_cast<const TB*>(a.B) + bz * a.sb_b;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int64_t k0 = 0; k0 < a.K; k0 += 16) {
    for (int i = threadIdx.x; i < 1024; i += 256) {
      const int r = i >> 4, kk = i & 15;
      const int64_t k = k0 + kk;
      const int64_t m = m0 + r, n = n0 + r;
      As[kk][r] = (m < a.M && k < a.K) ? to_f32(A[m * a.sa_m + k * a.sa_k]) : 0.f;
      Bs[kk][r] = (n < a.N && k < a.K) ? to_f32(B[n * a.sb_n + k * a.sb_k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  TC* C = static_cast<TC*>(a.C) + bz * a.sc_b;
  const TG* G = a.G ? static_cast<const TG*>(a.G) + bz * a.sg_b : nullptr;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty + 16 * i;
    if (m >= a.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx + 16 * j;
      if (n >= a.N) continue;
      float v = acc[i][j];
      if (a.sigmoid) v = 1.f / (1.f + expf(-v));
      if (G) v *= to_f32(G[m * a.sg_m + n * a.sg_n]);
      C[m * a.sc_m + n * a.sc_n] = from_f32<TC>(v);
    }
  }
}

template <typename TA, typename TB, typename TC, typename TG>
static int gemm_launch_t(const GemmArgs& a, cudaStream_t s) {
  if (a.M <= 0 || a.N <= 0 || a.batch <= 0) return MLA_OK;
  dim3 grid((unsigned)ceil_div(a.N, 64), (unsigned)ceil_div(a.M, 64), (unsigned)a.batch);
  if (grid.y > 65535u || grid.z > 65535u) return MLA_ERR_UNSUPPORTED;
  gemm_generic_kernel<TA, TB, TC, TG><<<grid, 256, 0, s>>>(a);
  MLA_LAUNCH_CHECK();
  return MLA_OK;
}

template <typename TA, typename TB, typename TC>
static int gemm_launch_g(const GemmArgs& a, int32_t g_dt, cudaStream_t s) {
  if (g_dt == MLA_BF16) return gemm_launch_t<TA, TB, TC, __nv_bfloat16>(a, s);
  return gemm_launch_t<TA, TB, TC, float>(a, s);
}

template <typename TA, typename TB>
static int gemm_launch_c(const GemmArgs& a, int32_t c_dt, int32_t g_dt, cudaStream_t s) {
  if (c_dt == MLA_BF16) return gemm_launch_g<TA, TB, __nv_bfloat16>(a, g_dt, s);
  return gemm_launch_g<TA, TB, float>(a, g_dt, s);
}

int gemm_generic(const GemmArgs& a, int32_t a_dt, int32_t b_dt, int32_t c_dt, int32_t g_dt,
                 cudaStream_t s) {
  if (a_dt == MLA_BF16 && b_dt == MLA_BF16) return gemm_launch_c<__nv_bfloat16, __nv_bfloat16>(a, c_dt, g_dt, s);
  if (a_dt == MLA_F32 && b_dt == MLA_BF16) return gemm_launch_c<float, __nv_bfloat16>(a, c_dt, g_dt, s);
  if (a_dt == MLA_BF16 && b_dt == MLA_F32) return gemm_launch_c<__nv_bfloat16, float>(a, c_dt, g_dt, s);
  return gemm_launch_c<float, float>(a, c_dt, g_dt, s);
}

// ---------------------------------------------------------------------------------------------
// strided row copy (e.g. q_pe into the tail of each absorbed query row)
// ---------------------------------------------------------------------------------------------
template <typename T>
__global__ void copy_rows_kernel(const T* __restrict__ src, int64_t ss, T* __restrict__ dst, int64_t ds,
                                 int64_t rows, int64_t cols) {
  const int64_t total = rows * cols;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / cols, c = e - r * cols;
    dst[r * ds + c] = src[r * ss + c];
  }
}

int copy_rows_strided(const void* src, int64_t ss, void* dst, int64_t ds, int64_t rows, int64_t cols,
                      int32_t dt, cudaStream_t s) {
  if (rows <= 0 || cols <= 0) return MLA_OK;
  const int64_t total = rows * cols;
  const unsigned blocks = (unsigned)std::min<int64_t>(ceil_div(total, 256), 4 * 148);
  if (dt == MLA_BF16)
    copy_rows_kernel<<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(src), ss,
                                            static_cast<__nv_bfloat16*>(dst), ds, rows, cols);
  else
    copy_rows_kernel<<<blocks, 256, 0, s>>>(static_cast<const float*>(src), ss,
                                            static_cast<float*>(dst), ds, rows, cols);
  MLA_LAUNCH_CHECK();
  return MLA_OK;
}

// ---------------------------------------------------------------------------------------------
// latent append: one CTA per new row; the row is built in fp32 shared memory, then stored in the
// cache dtype with 128-bit stores when the row pitch allows it
// ---------------------------------------------------------------------------------------------
// sine and cosine of the RoPE angle of pair i of a dr-wide rotary part at position pos:
// pos * theta^(-2i/d_r), computed and reduced to [-pi, pi] in double, so that the fp32 sine and cosine
// of the remainder keep full accuracy at positions of tens of thousands
__device__ __forceinline__ void rope_sincos(int32_t pos, int i, int dr, double log2_theta, float* sn, float* cs) {
  const double two_pi = 6.283185307179586476925286766559;
  const double ang = (double)pos * exp2(-2.0 * (double)i / (double)dr * log2_theta);
  const double turns = rint(ang * (1.0 / two_pi));
  sincosf((float)fma(-turns, two_pi, ang), sn, cs);
}

template <typename T>
__global__ void __launch_bounds__(128) append_latent_kernel(
    T* __restrict__ cache, const int64_t* __restrict__ row_idx, const float* __restrict__ c_new,
    int64_t c_stride, const float* __restrict__ kpe_new, int64_t kpe_stride,
    const int32_t* __restrict__ positions, int dc, int dr,
    uint32_t flags, float eps, double log2_theta, int vec8, int64_t cache_rows, int* status, float cache_scale) {
  extern __shared__ float row[];
  __shared__ float red[4];
  griddep_wait();
  griddep_launch_dependents();
  const int k = blockIdx.x;
  const int64_t target = row_idx[k];
  if (target < 0 || target >= cache_rows) {   // a row outside the cache is skipped and reported
    if (threadIdx.x == 0) atomicExch(status, (int)MLA_ERR_SHAPE);
    return;
  }
  const int W = dc + dr;
  float ss = 0.f;
  for (int i = threadIdx.x; i < dc; i += blockDim.x) {
    const float x = c_new[(int64_t)k * c_stride + i];
    row[i] = x;
    ss = fmaf(x, x, ss);
  }
  if (flags & MLA_APPEND_NORM) {
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    const float tot = red[0] + red[1] + red[2] + red[3];
    const float inv = 1.f / sqrtf(tot / (float)dc + eps);
    for (int i = threadIdx.x; i < dc; i += blockDim.x) row[i] *= inv;
  }
  if (dr > 0) {
    const int64_t kp = (int64_t)k * kpe_stride;
    if (flags & MLA_APPEND_ROPE) {
      const int32_t pos = positions[k];
      for (int i = threadIdx.x; i < dr / 2; i += blockDim.x) {
        float sn, cs;
        rope_sincos(pos, i, dr, log2_theta, &sn, &cs);
        const float x0 = kpe_new[kp + 2 * i], x1 = kpe_new[kp + 2 * i + 1];
        row[dc + 2 * i] = fmaf(x0, cs, -x1 * sn);
        row[dc + 2 * i + 1] = fmaf(x0, sn, x1 * cs);
      }
    } else {
      for (int i = threadIdx.x; i < dr; i += blockDim.x) row[dc + i] = kpe_new[kp + i];
    }
  }
  __syncthreads();
  T* dst = cache + target * (int64_t)W;
  if (vec8) {
    // 8 elements per thread per store: 16 B for bf16 (two 16 B stores for fp32)
    for (int i = threadIdx.x * 8; i < W; i += blockDim.x * 8) {
      if constexpr (sizeof(T) == 2) {
        uint4 v;
        __nv_bfloat162 p0 = __floats2bfloat162_rn(row[i], row[i + 1]);
        __nv_bfloat162 p1 = __floats2bfloat162_rn(row[i + 2], row[i + 3]);
        __nv_bfloat162 p2 = __floats2bfloat162_rn(row[i + 4], row[i + 5]);
        __nv_bfloat162 p3 = __floats2bfloat162_rn(row[i + 6], row[i + 7]);
        v.x = *reinterpret_cast<uint32_t*>(&p0);
        v.y = *reinterpret_cast<uint32_t*>(&p1);
        v.z = *reinterpret_cast<uint32_t*>(&p2);
        v.w = *reinterpret_cast<uint32_t*>(&p3);
        *reinterpret_cast<uint4*>(dst + i) = v;
      } else {
        *reinterpret_cast<float4*>(dst + i) = make_float4(row[i], row[i + 1], row[i + 2], row[i + 3]);
        *reinterpret_cast<float4*>(dst + i + 4) = make_float4(row[i + 4], row[i + 5], row[i + 6], row[i + 7]);
      }
    }
  } else if constexpr (sizeof(T) == 1) {
    // e4m3: the stored code is round-to-nearest-even of value / cache_scale (an IEEE fp32 division),
    // saturated to +-448
    for (int i = threadIdx.x; i < W; i += blockDim.x) dst[i] = from_f32<T>(row[i] / cache_scale);
  } else {
    for (int i = threadIdx.x; i < W; i += blockDim.x) dst[i] = from_f32<T>(row[i]);
  }
}

int append_latent_launch(const mla_dims& d, int32_t cache_dtype, void* cache, int64_t cache_rows,
                         const int64_t* row_idx, const float* c_new, const float* kpe_new,
                         const int32_t* positions, int64_t n_new, uint32_t flags, float eps,
                         float theta, cudaStream_t s) {
  return append_latent_strided(d, cache_dtype, cache, cache_rows, row_idx, c_new, d.kv_lora_rank, kpe_new,
                               d.rope_dim, positions, n_new, flags, eps, theta, s);
}

int append_latent_strided(const mla_dims& d, int32_t cache_dtype, void* cache, int64_t cache_rows,
                          const int64_t* row_idx, const float* c_new, int64_t c_stride, const float* kpe_new,
                          int64_t kpe_stride, const int32_t* positions, int64_t n_new, uint32_t flags,
                          float eps, float theta, cudaStream_t s, float cache_scale) {
  int* status = device_status_ptr();
  if (!status) return MLA_ERR_CUDA;
  if (n_new == 0) return MLA_OK;
  if (n_new > 0x7fffffff) return MLA_ERR_SHAPE;
  const int W = d.kv_lora_rank + d.rope_dim;
  const size_t es = dtype_bytes(cache_dtype);
  const int vec8 = cache_dtype != MLA_FP8_E4M3 && (W % 8 == 0) && aligned16(cache) && ((size_t)W * es) % 16 == 0;
  const size_t smem = (size_t)W * sizeof(float);
  if (smem > 48 * 1024) return MLA_ERR_UNSUPPORTED;
  if (cache_dtype == MLA_BF16)
    return launch_pdl(append_latent_kernel<__nv_bfloat16>, dim3((unsigned)n_new), dim3(128), smem, s,
                      static_cast<__nv_bfloat16*>(cache), row_idx, c_new, c_stride, kpe_new, kpe_stride,
                      positions, d.kv_lora_rank, d.rope_dim, flags, eps, log2((double)theta), vec8, cache_rows,
                      status, 1.f);
  if (cache_dtype == MLA_FP8_E4M3)
    return launch_pdl(append_latent_kernel<__nv_fp8_e4m3>, dim3((unsigned)n_new), dim3(128), smem, s,
                      static_cast<__nv_fp8_e4m3*>(cache), row_idx, c_new, c_stride, kpe_new, kpe_stride,
                      positions, d.kv_lora_rank, d.rope_dim, flags, eps, log2((double)theta), 0, cache_rows,
                      status, cache_scale);
  append_latent_kernel<float><<<(unsigned)n_new, 128, smem, s>>>(
      static_cast<float*>(cache), row_idx, c_new, c_stride, kpe_new, kpe_stride, positions, d.kv_lora_rank,
      d.rope_dim, flags, eps, log2((double)theta), vec8, cache_rows, status, 1.f);
  MLA_LAUNCH_CHECK();
  return MLA_OK;
}

// ---------------------------------------------------------------------------------------------
// rotary part of the queries: out[t, h, :] = R_{pos_t} src[t, h, :] (or a plain copy), fp32 in, the
// storage dtype out. Grid (token, chunk of 1024 pairs): the d_r/2 angles of the token once into shared
// memory, then 4 pairs per thread (two 16-byte loads, one 16-byte bf16 store when the row allows).
// ---------------------------------------------------------------------------------------------
constexpr int ROPE_PAIRS_PER_CTA = 1024;

template <typename T>
__global__ void __launch_bounds__(256) rope_rows_kernel(const float* __restrict__ src, T* __restrict__ out,
                                                        const int32_t* __restrict__ positions, int H, int dr,
                                                        int rotate, int vec, double log2_theta, int n_parts,
                                                        int64_t part_stride) {
  extern __shared__ float2 sc[];   // (sin, cos) of pair i
  griddep_wait();
  griddep_launch_dependents();
  const int t = blockIdx.x, half = dr / 2, pairs = H * half;
  const float2* row = reinterpret_cast<const float2*>(src + (int64_t)t * H * dr);
  T* o = out + (int64_t)t * H * dr;
  const int e0 = blockIdx.y * ROPE_PAIRS_PER_CTA + threadIdx.x * 4;
  // the source values are requested before the angles are formed (the two do not depend on each other)
  const bool vfast = vec && e0 + 3 < pairs;
  float4 u0 = make_float4(0.f, 0.f, 0.f, 0.f), u1 = u0;
  if (vfast) {
    // the source: one array, or the K-split partials of the projection that made it, added in order
    u0 = reinterpret_cast<const float4*>(row + e0)[0];
    u1 = reinterpret_cast<const float4*>(row + e0)[1];
    for (int q = 1; q < n_parts; ++q) {
      const float4* part = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(row + e0) + q * part_stride);
      const float4 a = part[0], b = part[1];
      u0.x += a.x; u0.y += a.y; u0.z += a.z; u0.w += a.w;
      u1.x += b.x; u1.y += b.y; u1.z += b.z; u1.w += b.w;
    }
  }
  if (rotate) {
    const int32_t pos = positions[t];
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
      float sn, cs;
      rope_sincos(pos, i, dr, log2_theta, &sn, &cs);
      sc[i] = make_float2(sn, cs);
    }
    __syncthreads();
  }
  auto turn = [&](float2 v, int e) {
    if (!rotate) return v;
    const float2 a = sc[e % half];
    return make_float2(fmaf(v.x, a.y, -v.y * a.x), fmaf(v.x, a.x, v.y * a.y));
  };
  if (vfast) {
    const float2 r0 = turn(make_float2(u0.x, u0.y), e0), r1 = turn(make_float2(u0.z, u0.w), e0 + 1);
    const float2 r2 = turn(make_float2(u1.x, u1.y), e0 + 2), r3 = turn(make_float2(u1.z, u1.w), e0 + 3);
    if constexpr (sizeof(T) == 2) {
      __nv_bfloat162 b0 = __floats2bfloat162_rn(r0.x, r0.y), b1 = __floats2bfloat162_rn(r1.x, r1.y);
      __nv_bfloat162 b2 = __floats2bfloat162_rn(r2.x, r2.y), b3 = __floats2bfloat162_rn(r3.x, r3.y);
      uint4 w;
      w.x = *reinterpret_cast<uint32_t*>(&b0); w.y = *reinterpret_cast<uint32_t*>(&b1);
      w.z = *reinterpret_cast<uint32_t*>(&b2); w.w = *reinterpret_cast<uint32_t*>(&b3);
      *reinterpret_cast<uint4*>(o + 2 * e0) = w;
    } else {
      reinterpret_cast<float4*>(o + 2 * e0)[0] = make_float4(r0.x, r0.y, r1.x, r1.y);
      reinterpret_cast<float4*>(o + 2 * e0)[1] = make_float4(r2.x, r2.y, r3.x, r3.y);
    }
    return;
  }
  for (int e = e0; e < min(e0 + 4, pairs); ++e) {
    float2 v = row[e];
    for (int q = 1; q < n_parts; ++q) {
      const float2 a = *reinterpret_cast<const float2*>(reinterpret_cast<const float*>(row + e) + q * part_stride);
      v.x += a.x; v.y += a.y;
    }
    const float2 r = turn(v, e);
    o[2 * e] = from_f32<T>(r.x);
    o[2 * e + 1] = from_f32<T>(r.y);
  }
}

int rope_rows_launch(int32_t dtype, const float* src, void* out, const int32_t* positions, int64_t n_rows, int H,
                     int dr, bool rotate, float theta, cudaStream_t s, int n_parts, int64_t part_stride) {
  if (n_rows <= 0 || dr <= 0) return MLA_OK;
  if (n_rows > 0x7fffffff || dr % 2) return MLA_ERR_SHAPE;
  const size_t smem = (size_t)(dr / 2) * sizeof(float2);
  if (smem > 48 * 1024) return MLA_ERR_UNSUPPORTED;
  const int64_t pairs = (int64_t)H * (dr / 2);
  const dim3 grid((unsigned)n_rows, (unsigned)ceil_div(pairs, ROPE_PAIRS_PER_CTA));
  if (grid.y > 65535u) return MLA_ERR_UNSUPPORTED;
  // 16-byte accesses: every row starts on 16 bytes in both buffers (src fp32 rows of H*dr floats; out
  // rows of H*dr elements) and each thread's 4 pairs do too
  const int vec = ((int64_t)H * dr) % 8 == 0 && aligned16(src) && aligned16(out) && (n_parts == 1 || part_stride % 4 == 0);
  const double l2t = log2((double)theta);
  if (dtype == MLA_BF16)
    return launch_pdl(rope_rows_kernel<__nv_bfloat16>, grid, dim3(256), smem, s, src,
                      static_cast<__nv_bfloat16*>(out), positions, H, dr, rotate ? 1 : 0, vec, l2t, n_parts,
                      part_stride);
  return launch_pdl(rope_rows_kernel<float>, grid, dim3(256), smem, s, src, static_cast<float*>(out), positions,
                    H, dr, rotate ? 1 : 0, vec, l2t, n_parts, part_stride);
}

// ---------------------------------------------------------------------------------------------
// merge of partial decode results by their log-sum-exp (split-KV across devices): part r holds the
// attention output O_r and lse_r of one query row and head over a disjoint slice of the positions;
//   m = max_r lse_r,  w_r = exp(lse_r - m),  O = sum_r w_r O_r / sum_r w_r,  lse = m + log sum_r w_r.
// One warp per (row, head); sums run over r in index order, so the result does not depend on timing.
// The parts may live in other devices' memory (peer pointers): the kernel only loads from them.
// ---------------------------------------------------------------------------------------------
constexpr int MERGE_GROUP = 2;   // parts whose columns one lane loads at once (64 registers: four blocks per SM)

struct MergeParts {
  const float* o[MLA_MERGE_MAX_PARTS];
  const float* l[MLA_MERGE_MAX_PARTS];
};

__global__ void __launch_bounds__(256) lse_merge_kernel(const __grid_constant__ MergeParts parts, int n_parts,
                                                        int64_t row0, int64_t n_rh, int H, int dc, int vec4,
                                                        float* __restrict__ out_lat, float* __restrict__ lse) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t x = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);   // local row * H + h
  if (x >= n_rh) return;
  const int64_t g = row0 * H + x;                                                    // global row * H + h
  // float4 rows of at most 512 columns: this lane's columns of the first MERGE_GROUP parts are requested
  // before the weights are known (every part is a whole [rows, H, d_c] buffer; an empty part's values
  // are loaded but never used), so that the weights' load and these overlap
  const bool fast = vec4 && dc % 128 == 0 && dc <= 512;
  const int ni = dc / 128;
  float4 v[MERGE_GROUP][4];
  if (fast) {
#pragma unroll
    for (int j = 0; j < MERGE_GROUP; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        v[j][i] = j < n_parts && i < ni ? *reinterpret_cast<const float4*>(parts.o[j] + g * dc + 4 * lane + 128 * i)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float lr = -INFINITY;
  if (lane < n_parts) lr = parts.l[lane][g];
  float m = lr;
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float* dst = out_lat + x * dc;
  if (m == -INFINITY) {                      // no part saw a position: empty attention
    for (int d = lane; d < dc; d += 32) dst[d] = 0.f;
    if (lane == 0 && lse) lse[x] = -INFINITY;
    return;
  }
  const float w_lane = lr == -INFINITY ? 0.f : expf(lr - m);
  float w[MLA_MERGE_MAX_PARTS];
  float wsum = 0.f;
#pragma unroll
  for (int r = 0; r < MLA_MERGE_MAX_PARTS; ++r) {
    w[r] = __shfl_sync(0xffffffffu, w_lane, r);
    if (r < n_parts) wsum += w[r];
  }
  const float inv = 1.f / wsum;
  if (fast) {
    // the lane's dc / 128 float4 columns, MERGE_GROUP parts at a time (one memory latency per group),
    // added up in part order as below
    float4 acc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r0 = 0; r0 < n_parts; r0 += MERGE_GROUP) {
      if (r0 > 0) {
#pragma unroll
        for (int j = 0; j < MERGE_GROUP; ++j) {
          const int r = r0 + j;
          const bool use = r < n_parts && __shfl_sync(0xffffffffu, w_lane, r & 31) != 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            v[j][i] = use && i < ni ? *reinterpret_cast<const float4*>(parts.o[r] + g * dc + 4 * lane + 128 * i)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int j = 0; j < MERGE_GROUP; ++j) {
        const int r = r0 + j;
        const float wr = __shfl_sync(0xffffffffu, w_lane, r & 31);
        if (r >= n_parts || wr == 0.f) continue;   // (an empty part's values take no part)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[i].x = fmaf(wr, v[j][i].x, acc[i].x); acc[i].y = fmaf(wr, v[j][i].y, acc[i].y);
          acc[i].z = fmaf(wr, v[j][i].z, acc[i].z); acc[i].w = fmaf(wr, v[j][i].w, acc[i].w);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (i < ni)
        *reinterpret_cast<float4*>(dst + 4 * lane + 128 * i) =
            make_float4(acc[i].x * inv, acc[i].y * inv, acc[i].z * inv, acc[i].w * inv);
  } else if (vec4) {
    for (int d = 4 * lane; d < dc; d += 128) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < MLA_MERGE_MAX_PARTS; ++r) {
        if (r >= n_parts) break;
        if (w[r] == 0.f) continue;               // (an empty part's output is not read)
        const float4 v = *reinterpret_cast<const float4*>(parts.o[r] + g * dc + d);
        acc.x = fmaf(w[r], v.x, acc.x); acc.y = fmaf(w[r], v.y, acc.y);
        acc.z = fmaf(w[r], v.z, acc.z); acc.w = fmaf(w[r], v.w, acc.w);
      }
      *reinterpret_cast<float4*>(dst + d) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
  } else {
    for (int d = lane; d < dc; d += 32) {
      float acc = 0.f;
      for (int r = 0; r < n_parts; ++r)
        if (w[r] != 0.f) acc = fmaf(w[r], parts.o[r][g * dc + d], acc);
      dst[d] = acc * inv;
    }
  }
  if (lane == 0 && lse) lse[x] = m + logf(wsum);
}

// ---------------------------------------------------------------------------------------------
// the index arrays of a decode step from host memory, carried in one launch's parameters (a kernel
// launch costs less than three small host-to-device copies, about 5 us each)
// ---------------------------------------------------------------------------------------------
constexpr int STEP_PARAM_BATCH = 240;   // keeps the parameter block under 4 KB
struct StepIndices {
  int32_t batch, has_pos;
  int32_t cu[STEP_PARAM_BATCH + 1];
  int32_t pos[STEP_PARAM_BATCH];
  int64_t rows[STEP_PARAM_BATCH];
};
static_assert(sizeof(StepIndices) <= 4000, "kernel parameter block");

__global__ void __launch_bounds__(256) put_step_indices_kernel(const __grid_constant__ StepIndices ix, int32_t* cu,
                                                               int64_t* rows, int32_t* pos) {
  griddep_wait();            // the previous step's kernels may still read these arrays
  griddep_launch_dependents();
  for (int i = threadIdx.x; i <= ix.batch; i += blockDim.x) cu[i] = ix.cu[i];
  for (int i = threadIdx.x; i < ix.batch; i += blockDim.x) {
    rows[i] = ix.rows[i];
    if (ix.has_pos) pos[i] = ix.pos[i];
  }
}

// MLA_ERR_UNSUPPORTED (nothing launched) above STEP_PARAM_BATCH sequences
int put_step_indices(const int32_t* cu_h, const int64_t* rows_h, const int32_t* pos_h, int batch, int32_t* cu,
                     int64_t* rows, int32_t* pos, cudaStream_t s) {
  if (batch < 0 || batch > STEP_PARAM_BATCH) return MLA_ERR_UNSUPPORTED;
  StepIndices ix;
  memset(&ix, 0, sizeof(ix));
  ix.batch = batch;
  ix.has_pos = pos_h ? 1 : 0;
  memcpy(ix.cu, cu_h, (size_t)(batch + 1) * sizeof(int32_t));
  memcpy(ix.rows, rows_h, (size_t)batch * sizeof(int64_t));
  if (pos_h) memcpy(ix.pos, pos_h, (size_t)batch * sizeof(int32_t));
  return launch_pdl(put_step_indices_kernel, dim3(1), dim3(256), 0, s, ix, cu, rows, pos);
}

int lse_merge_launch(int n_parts, const float* const* o_parts, const float* const* l_parts, int64_t row0,
                     int64_t n_rows, int H, int dc, float* out_lat, float* lse, cudaStream_t s) {
  if (n_rows <= 0) return MLA_OK;
  MergeParts mp{};
  bool aligned = aligned16(out_lat) && dc % 4 == 0;
  for (int r = 0; r < n_parts; ++r) {
    mp.o[r] = o_parts[r];
    mp.l[r] = l_parts[r];
    aligned = aligned && aligned16(o_parts[r]);
  }
  const int64_t n_rh = n_rows * H;
  const int64_t blocks = ceil_div(n_rh, 8);
  if (blocks > 0x7fffffffLL) return MLA_ERR_SHAPE;
  return launch_pdl(lse_merge_kernel, dim3((unsigned)blocks), dim3(256), 0, s, mp, n_parts, row0, n_rh, H, dc,
                    aligned ? 1 : 0, out_lat, lse);
}

// ---------------------------------------------------------------------------------------------
// split-KV absorbed decode on CUDA cores
//   grid: x = split of the positions, y = group of HG heads, z = query row (b * n_q + j)
//   per tile of DG_TP positions: stage the rows in shared memory (fp32), scores for every
//   (head, position), per-head online softmax by one warp (shuffle max / sum), O update in
//   registers (HG * d_c accumulators spread over the block)
// ---------------------------------------------------------------------------------------------
constexpr int DG_THREADS = 256;
constexpr int DG_TP = 32;
constexpr int DG_MAXE = 32;  // accumulators per thread: HG * d_c <= DG_THREADS * DG_MAXE

struct DecodeGenericParams {
  const void* q_abs; const void* cache; const int32_t* cu;
  int n_q, H, dc, W, HG, chunk, n_splits;
  float scale; int causal;
  float* out_lat; float* lse;            // used when n_splits == 1
  float* o_part; float* m_part; float* l_part;   // [split][row][H](*dc)
  int64_t rows;
  int64_t total_rows;
  float cache_scale;                     // cache element times this = the value (1 unless e4m3)
};

template <typename T, typename TC = T>
__global__ void __launch_bounds__(DG_THREADS) decode_generic_kernel(DecodeGenericParams p) {
  extern __shared__ float sm[];
  const int W = p.W, HG = p.HG;
  float* qs = sm;                          // [HG][W]
  float* Ks = qs + HG * W;                 // [DG_TP][W + 1]
  float* Ps = Ks + DG_TP * (W + 1);        // [HG][DG_TP]
  float* ms = Ps + HG * DG_TP;             // [HG]
  float* ls = ms + HG;                     // [HG]
  float* cs = ls + HG;                     // [HG]

  const int split = blockIdx.x;
  const int h0 = blockIdx.y * HG;
  const int64_t row = blockIdx.z;
  const int b = (int)(row / p.n_q), j = (int)(row % p.n_q);
  // sequence bounds, clamped to the cache so that a malformed cu_seqlens cannot read outside it
  const int64_t c0 = p.cu[b], c1 = p.cu[b + 1];
  const int64_t start = c0 < 0 ? 0 : (c0 > p.total_rows ? p.total_rows : c0);
  const int64_t stop = c1 < start ? start : (c1 > p.total_rows ? p.total_rows : c1);
  const int Tb = (int)(stop - start);
  int cnt = p.causal ? (Tb - p.n_q + j + 1) : Tb;
  cnt = max(0, min(cnt, Tb));
  const int lo = split * p.chunk;
  const int hi = min(lo + p.chunk, cnt);
  const int hg = min(HG, p.H - h0);

  const T* q = static_cast<const T*>(p.q_abs) + (row * p.H + h0) * (int64_t)W;
  for (int e = threadIdx.x; e < hg * W; e += DG_THREADS) qs[e] = to_f32(q[e]);
  for (int hh = threadIdx.x; hh < HG; hh += DG_THREADS) { ms[hh] = -INFINITY; ls[hh] = 0.f; }
  float o[DG_MAXE];
#pragma unroll
  for (int i = 0; i < DG_MAXE; ++i) o[i] = 0.f;
  const int n_el = hg * p.dc;
  __syncthreads();

  const TC* cache = static_cast<const TC*>(p.cache);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t0 = lo; t0 < hi; t0 += DG_TP) {
    const int nt = min(DG_TP, hi - t0);
    for (int e = threadIdx.x; e < nt * W; e += DG_THREADS) {
      const int tt = e / W, k = e - tt * W;
      Ks[tt * (W + 1) + k] = to_f32(cache[(start + t0 + tt) * (int64_t)W + k]) * p.cache_scale;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < hg * DG_TP; e += DG_THREADS) {
      const int hh = e / DG_TP, tt = e - hh * DG_TP;
      float s = -INFINITY;
      if (tt < nt) {
        const float* qa = qs + hh * W;
        const float* ka = Ks + tt * (W + 1);
        float acc = 0.f;
        for (int k = 0; k < W; ++k) acc = fmaf(qa[k], ka[k], acc);
        s = acc * p.scale;
      }
      Ps[e] = s;
    }
    __syncthreads();
    for (int hh = warp; hh < hg; hh += DG_THREADS / 32) {
      const float s = Ps[hh * DG_TP + lane];
      float mt = s;
      for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float m_old = ms[hh];
      const float m_new = fmaxf(m_old, mt);
      const float pr = (s == -INFINITY) ? 0.f : expf(s - m_new);
      float sum = pr;
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      Ps[hh * DG_TP + lane] = pr;
      __syncwarp();
      if (lane == 0) {
        const float c = (m_old == -INFINITY) ? 0.f : expf(m_old - m_new);
        ls[hh] = ls[hh] * c + sum;
        ms[hh] = m_new;
        cs[hh] = c;
      }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < DG_MAXE; ++i) {
      const int e = threadIdx.x + i * DG_THREADS;
      if (e < n_el) {
        const int hh = e / p.dc, d = e - hh * p.dc;
        float acc = o[i] * cs[hh];
        const float* pp = Ps + hh * DG_TP;
        for (int tt = 0; tt < nt; ++tt) acc = fmaf(pp[tt], Ks[tt * (W + 1) + d], acc);
        o[i] = acc;
      }
    }
    __syncthreads();
  }

  if (p.n_splits == 1) {
#pragma unroll
    for (int i = 0; i < DG_MAXE; ++i) {
      const int e = threadIdx.x + i * DG_THREADS;
      if (e < n_el) {
        const int hh = e / p.dc, d = e - hh * p.dc;
        const float l = ls[hh];
        p.out_lat[(row * p.H + h0 + hh) * (int64_t)p.dc + d] = l > 0.f ? o[i] / l : 0.f;
      }
    }
    if (p.lse)
      for (int hh = threadIdx.x; hh < hg; hh += DG_THREADS) {
        const float l = ls[hh];
        p.lse[row * p.H + h0 + hh] = l > 0.f ? ms[hh] + logf(l) : -INFINITY;
      }
  } else {
    const int64_t base = ((int64_t)split * p.rows + row) * p.H + h0;
#pragma unroll
    for (int i = 0; i < DG_MAXE; ++i) {
      const int e = threadIdx.x + i * DG_THREADS;
      if (e < n_el) {
        const int hh = e / p.dc, d = e - hh * p.dc;
        p.o_part[(base + hh) * p.dc + d] = o[i];
      }
    }
    for (int hh = threadIdx.x; hh < hg; hh += DG_THREADS) {
      p.m_part[base + hh] = ms[hh];
      p.l_part[base + hh] = ls[hh];
    }
  }
}

// merge of split partials: one CTA per (row, head); out = sum_s w_s O_s / sum_s w_s l_s with
// w_s = exp(m_s - max_s m_s)
__global__ void decode_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ m_part,
                                      const float* __restrict__ l_part, int n_splits, int64_t rh,
                                      int dc, float* __restrict__ out_lat, float* __restrict__ lse) {
  const int64_t x = blockIdx.x;  // row * H + h
  float M = -INFINITY;
  for (int s = 0; s < n_splits; ++s) M = fmaxf(M, m_part[s * rh + x]);
  float L = 0.f;
  for (int s = 0; s < n_splits; ++s) {
    const float m = m_part[s * rh + x];
    if (m != -INFINITY) L += expf(m - M) * l_part[s * rh + x];
  }
  for (int d = threadIdx.x; d < dc; d += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < n_splits; ++s) {
      const float m = m_part[s * rh + x];
      if (m != -INFINITY) acc += expf(m - M) * o_part[(s * rh + x) * dc + d];
    }
    out_lat[x * dc + d] = L > 0.f ? acc / L : 0.f;
  }
  if (lse && threadIdx.x == 0) lse[x] = L > 0.f ? M + logf(L) : -INFINITY;
}

struct GenericPlan { int HG, chunk, n_splits; size_t smem, ws; };

static GenericPlan plan_generic(const DecodeArgs& a) {
  GenericPlan g;
  const int W = a.dc + a.dr;
  g.HG = std::max(1, std::min<int>(a.H, (DG_THREADS * DG_MAXE) / std::max(1, a.dc)));
  const int64_t rows = (int64_t)a.batch * a.n_q;
  const int64_t base = rows * ceil_div(a.H, g.HG);
  const int64_t want = 2LL * sm_count();
  int64_t splits = std::max<int64_t>(1, ceil_div(want, std::max<int64_t>(1, base)));
  const int64_t max_tiles = std::max<int64_t>(1, ceil_div(a.max_seqlen, DG_TP));
  splits = std::min(splits, max_tiles);
  int64_t chunk = ceil_div(std::max<int64_t>(a.max_seqlen, 1), splits);
  chunk = ceil_div(chunk, DG_TP) * DG_TP;
  splits = std::max<int64_t>(1, ceil_div(std::max<int64_t>(a.max_seqlen, 1), chunk));
  g.chunk = (int)chunk;
  g.n_splits = (int)splits;
  g.smem = sizeof(float) * ((size_t)g.HG * W + (size_t)DG_TP * (W + 1) + (size_t)g.HG * DG_TP + 3 * (size_t)g.HG);
  g.ws = 0;
  if (g.n_splits > 1) {
    const size_t rh = (size_t)rows * a.H;
    g.ws = round_up(sizeof(float) * (size_t)g.n_splits * rh * a.dc, 256) +
           2 * round_up(sizeof(float) * (size_t)g.n_splits * rh, 256);
  }
  return g;
}

size_t decode_generic_workspace(const DecodeArgs& a) { return plan_generic(a).ws; }

template <typename T, typename TC>
static int decode_generic_run(const DecodeGenericParams& p, dim3 grid, size_t smem, cudaStream_t s) {
  if (cudaFuncSetAttribute(decode_generic_kernel<T, TC>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return MLA_ERR_CUDA;
  decode_generic_kernel<T, TC><<<grid, DG_THREADS, smem, s>>>(p);
  MLA_LAUNCH_CHECK();
  return MLA_OK;
}

int decode_generic_launch(const DecodeArgs& a, int32_t dtype, cudaStream_t s, int32_t cache_dtype) {
  const GenericPlan g = plan_generic(a);
  const int64_t rows = (int64_t)a.batch * a.n_q;
  if (rows == 0) return MLA_OK;
  if (g.smem > 200 * 1024) return MLA_ERR_UNSUPPORTED;
  if (a.workspace_bytes < g.ws || (g.ws && !a.workspace)) return MLA_ERR_WORKSPACE;
  DecodeGenericParams p;
  p.q_abs = a.q_abs; p.cache = a.cache; p.cu = a.cu_seqlens;
  p.n_q = a.n_q; p.H = a.H; p.dc = a.dc; p.W = a.dc + a.dr; p.HG = g.HG;
  p.chunk = g.chunk; p.n_splits = g.n_splits; p.scale = a.scale; p.causal = a.causal ? 1 : 0;
  p.out_lat = a.out_lat; p.lse = a.lse; p.rows = rows; p.total_rows = a.total_rows;
  p.cache_scale = cache_dtype == MLA_FP8_E4M3 ? a.cache_scale : 1.f;
  const size_t rh = (size_t)rows * a.H;
  char* ws = static_cast<char*>(a.workspace);
  p.o_part = reinterpret_cast<float*>(ws);
  p.m_part = reinterpret_cast<float*>(ws + round_up(sizeof(float) * (size_t)g.n_splits * rh * a.dc, 256));
  p.l_part = p.m_part + round_up(sizeof(float) * (size_t)g.n_splits * rh, 256) / sizeof(float);
  dim3 grid((unsigned)g.n_splits, (unsigned)ceil_div(a.H, g.HG), (unsigned)rows);
  if (grid.y > 65535u || grid.z > 65535u) return MLA_ERR_UNSUPPORTED;
  int st;
  if (cache_dtype == MLA_FP8_E4M3)
    st = dtype == MLA_BF16 ? decode_generic_run<__nv_bfloat16, __nv_fp8_e4m3>(p, grid, g.smem, s)
                           : decode_generic_run<float, __nv_fp8_e4m3>(p, grid, g.smem, s);
  else
    st = dtype == MLA_BF16 ? decode_generic_run<__nv_bfloat16, __nv_bfloat16>(p, grid, g.smem, s)
                           : decode_generic_run<float, float>(p, grid, g.smem, s);
  if (st) return st;
  if (g.n_splits > 1) {
    decode_combine_kernel<<<(unsigned)rh, 128, 0, s>>>(p.o_part, p.m_part, p.l_part, g.n_splits,
                                                       (int64_t)rh, a.dc, a.out_lat, a.lse);
    MLA_LAUNCH_CHECK();
  }
  return MLA_OK;
}

}  // namespace mla
