// mla_api.cu -- the C ABI declared in include/mla.h: host-side validation and kernel dispatch.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "tc.cuh"

namespace mla {
// generic.cu: the step's index arrays written into the workspace by one kernel whose launch parameters
// carry them (MLA_ERR_UNSUPPORTED, nothing launched, for more sequences than that kernel takes)
int put_step_indices(const int32_t* cu_h, const int64_t* rows_h, const int32_t* pos_h, int batch, int32_t* cu,
                     int64_t* rows, int32_t* pos, cudaStream_t s);
}  // namespace mla

using namespace mla;

namespace {

bool dtype_ok(int32_t dt) { return dt == MLA_F32 || dt == MLA_BF16; }

int check_dims(const mla_dims* d) {
  if (!d) return MLA_ERR_NULL;
  if (d->n_heads <= 0 || d->kv_lora_rank <= 0 || d->rope_dim < 0 || d->qk_nope < 0 ||
      d->v_head < 0 || d->d_model < 0)
    return MLA_ERR_SHAPE;
  if (!(d->kq_scale >= 0.f) || isinf(d->kq_scale)) return MLA_ERR_SHAPE;
  return MLA_OK;
}

float effective_scale(const mla_dims* d) {
  if (d->kq_scale > 0.f) return d->kq_scale;
  const int w = d->qk_nope + d->rope_dim;
  return w > 0 ? 1.0f / sqrtf((float)w) : 1.0f;
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// A second stream per device for work of a call that may overlap the rest of it, with the two events
// that fork it from the caller's stream and join it back; the mutex keeps the record / wait pairs of
// concurrent calls on one device from interleaving. Created on first use, kept for the process.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  std::mutex m;
};

SideStream* side_stream() {
  static SideStream sides[64];
  static std::mutex create;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SideStream* x = &sides[dev];
  std::lock_guard<std::mutex> lock(create);
  if (!x->s) {
    cudaStream_t st = nullptr;
    cudaEvent_t f = nullptr, j = nullptr;
    if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&f, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&j, cudaEventDisableTiming) != cudaSuccess) {
      (void)cudaGetLastError();
      if (f) cudaEventDestroy(f);
      if (st) cudaStreamDestroy(st);
      return nullptr;
    }
    x->fork = f;
    x->join = j;
    x->s = st;
  }
  return x;
}

// bf16 operands of the tensor-core kernels are read with 16-byte vector or TMA accesses
int check_align(int32_t dt, std::initializer_list<const void*> ptrs) {
  if (dt != MLA_BF16) {
    for (const void* p : ptrs)
      if (p && (reinterpret_cast<uintptr_t>(p) & 3u)) return MLA_ERR_ALIGN;
    return MLA_OK;
  }
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MLA_ERR_ALIGN;
  return MLA_OK;
}

}  // namespace

extern "C" {

const char* mla_status_string(int32_t s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_NULL: return "MLA_ERR_NULL: a required pointer is NULL";
    case MLA_ERR_SHAPE: return "MLA_ERR_SHAPE: invalid or inconsistent sizes";
    case MLA_ERR_DTYPE: return "MLA_ERR_DTYPE: unknown or unsupported dtype";
    case MLA_ERR_ALIGN: return "MLA_ERR_ALIGN: pointer not aligned as required";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE: workspace missing or too small";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA: a CUDA call or kernel launch failed";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT: a bounded device wait gave up";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED: request not implemented by this build";
    case MLA_ERR_MODE: return "MLA_ERR_MODE: unknown mode or flag";
    default: return "unknown mla status";
  }
}

int32_t mla_abi_version(void) { return 3; }

int32_t mla_append_latent(const mla_dims* dims, int32_t cache_dtype, void* cache, int64_t cache_rows,
                          const int64_t* row_idx, const float* c_new, const float* kpe_new,
                          const int32_t* positions, int64_t n_new, uint32_t flags, float eps,
                          float rope_theta, void* stream) {
  int st = check_dims(dims);
  if (st) return st;
  if (!dtype_ok(cache_dtype)) return MLA_ERR_DTYPE;
  if (flags & ~(uint32_t)(MLA_APPEND_NORM | MLA_APPEND_ROPE)) return MLA_ERR_MODE;
  if (n_new < 0 || cache_rows < 0) return MLA_ERR_SHAPE;
  if (n_new == 0) return MLA_OK;
  if (!cache || !row_idx || !c_new) return MLA_ERR_NULL;
  if (dims->rope_dim > 0 && !kpe_new) return MLA_ERR_NULL;
  if ((flags & MLA_APPEND_ROPE) && dims->rope_dim > 0) {
    if (!positions) return MLA_ERR_NULL;
    if (dims->rope_dim % 2) return MLA_ERR_SHAPE;
    if (!(rope_theta > 0.f)) return MLA_ERR_SHAPE;
  }
  if ((flags & MLA_APPEND_NORM) && !(eps >= 0.f)) return MLA_ERR_SHAPE;
  return append_latent_launch(*dims, cache_dtype, cache, cache_rows, row_idx, c_new, kpe_new, positions, n_new,
                              flags, eps, rope_theta, as_stream(stream));
}

int32_t mla_append_latent_fp8(const mla_dims* dims, uint8_t* cache, int64_t cache_rows, const int64_t* row_idx,
                              const float* c_new, const float* kpe_new, const int32_t* positions, int64_t n_new,
                              uint32_t flags, float eps, float rope_theta, float cache_scale, void* stream) {
  int st = check_dims(dims);
  if (st) return st;
  if (flags & ~(uint32_t)(MLA_APPEND_NORM | MLA_APPEND_ROPE)) return MLA_ERR_MODE;
  if (n_new < 0 || cache_rows < 0) return MLA_ERR_SHAPE;
  if (!(cache_scale > 0.f) || isinf(cache_scale)) return MLA_ERR_SHAPE;
  if (n_new == 0) return MLA_OK;
  if (!cache || !row_idx || !c_new) return MLA_ERR_NULL;
  if (dims->rope_dim > 0 && !kpe_new) return MLA_ERR_NULL;
  if ((flags & MLA_APPEND_ROPE) && dims->rope_dim > 0) {
    if (!positions) return MLA_ERR_NULL;
    if (dims->rope_dim % 2) return MLA_ERR_SHAPE;
    if (!(rope_theta > 0.f)) return MLA_ERR_SHAPE;
  }
  if ((flags & MLA_APPEND_NORM) && !(eps >= 0.f)) return MLA_ERR_SHAPE;
  return append_latent_strided(*dims, MLA_FP8_E4M3, cache, cache_rows, row_idx, c_new, dims->kv_lora_rank, kpe_new,
                               dims->rope_dim, positions, n_new, flags, eps, rope_theta, as_stream(stream),
                               cache_scale);
}

int32_t mla_absorb_weights(const mla_dims* dims, int32_t dtype, int32_t mode, const void* x,
                           const void* x_pe, const void* w, int64_t n_rows, void* out, void* stream) {
  int st = check_dims(dims);
  if (st) return st;
  if (!dtype_ok(dtype)) return MLA_ERR_DTYPE;
  if (n_rows < 0) return MLA_ERR_SHAPE;
  const int64_t H = dims->n_heads, dc = dims->kv_lora_rank, dr = dims->rope_dim;
  const int64_t n = dims->qk_nope, dv = dims->v_head, D = dims->d_model;
  cudaStream_t s = as_stream(stream);
  if (mode == MLA_ABSORB_QUERY) {
    if (n_rows == 0) return MLA_OK;
    if (!x || !w || !out || (dr > 0 && !x_pe)) return MLA_ERR_NULL;
    if (n <= 0) return MLA_ERR_SHAPE;
    if ((st = check_align(dtype, {x, x_pe, w, out}))) return st;
    const int64_t W = dc + dr;
    if (dtype == MLA_BF16 && tc_absorb_supported(*dims, n_rows))
      return tc_absorb_query(*dims, x, x_pe, w, n_rows, out, s);
    // out[t,h,j] = sum_i x[t,h,i] w[h,i,j]: batch = h, M = t, N = j, K = i
    GemmArgs g{};
    g.A = x;   g.sa_b = n;  g.sa_m = H * n;  g.sa_k = 1;
    g.B = w;   g.sb_b = n * dc; g.sb_n = 1;  g.sb_k = dc;
    g.C = out; g.sc_b = W;  g.sc_m = H * W;  g.sc_n = 1;
    g.M = n_rows; g.N = dc; g.K = n; g.batch = H;
    if ((st = gemm_generic(g, dtype, dtype, dtype, dtype, s))) return st;
    if (dr > 0) {
      // q_pe rows [n_rows * H, dr] into the tail of each absorbed row
      if ((st = copy_rows_strided(x_pe, dr, static_cast<char*>(out) + dc * dtype_bytes(dtype), W,
                                  n_rows * H, dr, dtype, s)))
        return st;
    }
    return MLA_OK;
  }
  if (mode == MLA_FOLD_QK) {
    if (n_rows == 0) return MLA_OK;
    if (!x || !w || !out) return MLA_ERR_NULL;
    if (n <= 0) return MLA_ERR_SHAPE;
    // out[h] = x[h] . w[h]^T: x [H, R, n], w [H, dc, n], out [H, R, dc]
    GemmArgs g{};
    g.A = x;   g.sa_b = n_rows * n; g.sa_m = n;  g.sa_k = 1;
    g.B = w;   g.sb_b = dc * n;     g.sb_n = n;  g.sb_k = 1;
    g.C = out; g.sc_b = n_rows * dc; g.sc_m = dc; g.sc_n = 1;
    g.M = n_rows; g.N = dc; g.K = n; g.batch = H;
    return gemm_generic(g, dtype, dtype, dtype, dtype, s);
  }
  if (mode == MLA_FOLD_VO) {
    if (!x || !w || !out) return MLA_ERR_NULL;
    if (n_rows != dc || dv <= 0 || D <= 0) return MLA_ERR_SHAPE;
    // out[h] = x[h] . w[h]: x [H, dc, dv], w [H, dv, D], out [H, dc, D]
    GemmArgs g{};
    g.A = x;   g.sa_b = dc * dv; g.sa_m = dv; g.sa_k = 1;
    g.B = w;   g.sb_b = dv * D;  g.sb_n = 1;  g.sb_k = D;
    g.C = out; g.sc_b = dc * D;  g.sc_m = D;  g.sc_n = 1;
    g.M = dc; g.N = D; g.K = dv; g.batch = H;
    return gemm_generic(g, dtype, dtype, dtype, dtype, s);
  }
  return MLA_ERR_MODE;
}

static DecodeArgs make_decode_args(const mla_dims* d, int32_t batch, int32_t n_q, int64_t max_seqlen,
                                   int64_t total_rows, uint32_t flags) {
  DecodeArgs a{};
  a.batch = batch; a.n_q = n_q; a.H = d->n_heads; a.dc = d->kv_lora_rank; a.dr = d->rope_dim;
  a.max_seqlen = max_seqlen; a.total_rows = total_rows;
  a.scale = effective_scale(d);
  a.causal = (flags & MLA_DECODE_CAUSAL) != 0;
  return a;
}

static int check_decode_sizes(const mla_dims* dims, int32_t dtype, int32_t batch, int32_t n_q,
                              int64_t max_seqlen, int64_t total_rows, uint32_t flags) {
  int st = check_dims(dims);
  if (st) return st;
  if (!dtype_ok(dtype)) return MLA_ERR_DTYPE;
  if (flags & ~(uint32_t)(MLA_DECODE_CAUSAL | MLA_DECODE_OUT_BF16)) return MLA_ERR_MODE;
  if (batch < 0 || n_q <= 0 || max_seqlen < 0 || total_rows < 0) return MLA_ERR_SHAPE;
  if (max_seqlen > 0x7fffffffLL || total_rows > 0x7fffffffLL) return MLA_ERR_SHAPE;
  if ((int64_t)batch * max_seqlen < total_rows) return MLA_ERR_SHAPE;
  if ((flags & MLA_DECODE_CAUSAL) && batch > 0 && max_seqlen < n_q) return MLA_ERR_SHAPE;
  return MLA_OK;
}

int32_t mla_decode_workspace_size(const mla_dims* dims, int32_t dtype, int32_t batch, int32_t n_q,
                                  int64_t max_seqlen, int64_t total_rows, uint32_t flags,
                                  size_t* bytes) {
  if (!bytes) return MLA_ERR_NULL;
  // MLA_FP8_E4M3: the scratch of mla_decode_absorbed_fp8 (whatever the query's dtype)
  const bool fp8 = dtype == MLA_FP8_E4M3;
  int st = check_decode_sizes(dims, fp8 ? MLA_F32 : dtype, batch, n_q, max_seqlen, total_rows, flags);
  if (st) return st;
  DecodeArgs a = make_decode_args(dims, batch, n_q, max_seqlen, total_rows, flags);
  if (fp8) {
    // the CUDA-core decode (an fp32 query) or the tensor-core one (a bf16 query): room for either
    a.cache_f8 = true;
    *bytes = decode_generic_workspace(a);
    if (tc_decode_supported(a)) *bytes = std::max(*bytes, tc_decode_workspace(a));
  }
  else if (dtype == MLA_BF16 && tc_decode_supported(a))
    *bytes = tc_decode_workspace(a);
  else
    *bytes = decode_generic_workspace(a);
  return MLA_OK;
}

int32_t mla_decode_absorbed(const mla_dims* dims, int32_t dtype, const void* q_abs, const void* cache,
                            const int32_t* cu_seqlens, int32_t batch, int32_t n_q, int64_t max_seqlen,
                            int64_t total_rows, uint32_t flags, float* out_lat, float* lse,
                            void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_decode_sizes(dims, dtype, batch, n_q, max_seqlen, total_rows, flags);
  if (st) return st;
  if (batch == 0) return MLA_OK;
  if (!q_abs || !cu_seqlens || !out_lat || (total_rows > 0 && !cache)) return MLA_ERR_NULL;
  if ((st = check_align(dtype, {q_abs, cache, out_lat, lse}))) return st;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return MLA_ERR_ALIGN;
  DecodeArgs a = make_decode_args(dims, batch, n_q, max_seqlen, total_rows, flags);
  a.q_abs = q_abs; a.cache = cache; a.cu_seqlens = cu_seqlens;
  a.out_lat = out_lat; a.lse = lse; a.workspace = workspace; a.workspace_bytes = workspace_bytes;
  cudaStream_t s = as_stream(stream);
  if (flags & MLA_DECODE_OUT_BF16) a.out_lat_bf16 = out_lat;
  if (dtype == MLA_BF16 && tc_decode_supported(a)) {
    if (workspace_bytes < tc_decode_workspace(a) || !workspace) return MLA_ERR_WORKSPACE;
    return tc_decode_launch(a, s);
  }
  if (flags & MLA_DECODE_OUT_BF16) return MLA_ERR_UNSUPPORTED;   // the tensor-core route only
  if (workspace_bytes < decode_generic_workspace(a)) return MLA_ERR_WORKSPACE;
  return decode_generic_launch(a, dtype, s);
}

int32_t mla_decode_absorbed_fp8(const mla_dims* dims, int32_t q_dtype, const void* q_abs, const uint8_t* cache,
                                float cache_scale, const int32_t* cu_seqlens, int32_t batch, int32_t n_q,
                                int64_t max_seqlen, int64_t total_rows, uint32_t flags, float* out_lat, float* lse,
                                void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_decode_sizes(dims, q_dtype, batch, n_q, max_seqlen, total_rows, flags);
  if (st) return st;
  if (!(cache_scale > 0.f) || isinf(cache_scale)) return MLA_ERR_SHAPE;
  if (batch == 0) return MLA_OK;
  if (!q_abs || !cu_seqlens || !out_lat || (total_rows > 0 && !cache)) return MLA_ERR_NULL;
  if ((st = check_align(q_dtype, {q_abs})) || (reinterpret_cast<uintptr_t>(out_lat) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return st ? st : MLA_ERR_ALIGN;
  DecodeArgs a = make_decode_args(dims, batch, n_q, max_seqlen, total_rows, flags);
  a.q_abs = q_abs; a.cache = cache; a.cu_seqlens = cu_seqlens;
  a.out_lat = out_lat; a.lse = lse; a.workspace = workspace; a.workspace_bytes = workspace_bytes;
  a.cache_scale = cache_scale;
  a.cache_f8 = true;
  if (flags & MLA_DECODE_OUT_BF16) {
    if (reinterpret_cast<uintptr_t>(out_lat) & 15u) return MLA_ERR_ALIGN;
    a.out_lat_bf16 = out_lat;
  }
  if (q_dtype == MLA_BF16 && tc_decode_supported(a)) {
    if (workspace_bytes < tc_decode_workspace(a) || !workspace) return MLA_ERR_WORKSPACE;
    return tc_decode_launch(a, as_stream(stream));
  }
  if (flags & MLA_DECODE_OUT_BF16) return MLA_ERR_UNSUPPORTED;   // the tensor-core route only
  if (workspace_bytes < decode_generic_workspace(a)) return MLA_ERR_WORKSPACE;
  return decode_generic_launch(a, q_dtype, as_stream(stream), MLA_FP8_E4M3);
}

int32_t mla_out_project_workspace_size(const mla_dims* dims, int32_t dtype, int64_t n_rows,
                                       size_t* bytes) {
  if (!bytes) return MLA_ERR_NULL;
  int st = check_dims(dims);
  if (st) return st;
  if (!dtype_ok(dtype)) return MLA_ERR_DTYPE;
  if (n_rows < 0) return MLA_ERR_SHAPE;
  // v [n_rows, H * v_head] in dtype, plus the tensor-core path's own scratch
  size_t b = round_up((size_t)n_rows * dims->n_heads * dims->v_head * dtype_bytes(dtype), 256);
  if (dtype == MLA_BF16) b += tc_out_project_extra_workspace(*dims, n_rows);
  *bytes = b;
  return MLA_OK;
}

}  // extern "C"

// out_lat in fp32 (lat_bf16 false) or bf16 (the tensor-core decode's MLA_DECODE_OUT_BF16 output)
static int32_t out_project_impl(const mla_dims* dims, int32_t dtype, const void* out_lat, bool lat_bf16,
                                const void* w_uv, const void* w_o, const void* gate, int64_t n_rows, void* y,
                                void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_dims(dims);
  if (st) return st;
  if (!dtype_ok(dtype)) return MLA_ERR_DTYPE;
  if (n_rows < 0) return MLA_ERR_SHAPE;
  if (n_rows == 0) return MLA_OK;
  if (!out_lat || !w_uv || !w_o || !y) return MLA_ERR_NULL;
  const int64_t H = dims->n_heads, dc = dims->kv_lora_rank, dv = dims->v_head, D = dims->d_model;
  if (dv <= 0 || D <= 0) return MLA_ERR_SHAPE;
  size_t need = 0;
  if ((st = mla_out_project_workspace_size(dims, dtype, n_rows, &need))) return st;
  if (!workspace || workspace_bytes < need) return MLA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return MLA_ERR_ALIGN;
  if ((st = check_align(dtype, {w_uv, w_o, gate, y}))) return st;
  if (reinterpret_cast<uintptr_t>(out_lat) & 15u) return MLA_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  void* v = workspace;
  if (dtype == MLA_BF16 && tc_out_project_supported(*dims, n_rows))
    return tc_out_project(*dims, out_lat, lat_bf16, w_uv, w_o, gate, n_rows, y, workspace, workspace_bytes, s);
  // stage 1: v[t, h, i] = gate * sum_j out_lat[t, h, j] W_UV[h, i, j]; batch = h, M = t, N = i
  GemmArgs g{};
  g.A = out_lat; g.sa_b = dc; g.sa_m = H * dc; g.sa_k = 1;
  g.B = w_uv;    g.sb_b = dv * dc; g.sb_n = dc; g.sb_k = 1;
  g.C = v;       g.sc_b = dv; g.sc_m = H * dv; g.sc_n = 1;
  g.G = gate;    g.sg_b = dv; g.sg_m = H * dv; g.sg_n = 1;
  g.M = n_rows; g.N = dv; g.K = dc; g.batch = H;
  if ((st = gemm_generic(g, lat_bf16 ? MLA_BF16 : MLA_F32, dtype, dtype, dtype, s))) return st;
  // stage 2: y[t, d] = sum_k v[t, k] W_O[d, k]
  GemmArgs o{};
  o.A = v;   o.sa_b = 0; o.sa_m = H * dv; o.sa_k = 1;
  o.B = w_o; o.sb_b = 0; o.sb_n = H * dv; o.sb_k = 1;
  o.C = y;   o.sc_b = 0; o.sc_m = D; o.sc_n = 1;
  o.M = n_rows; o.N = D; o.K = H * dv; o.batch = 1;
  return gemm_generic(o, dtype, dtype, dtype, dtype, s);
}

extern "C" {

int32_t mla_out_project(const mla_dims* dims, int32_t dtype, const float* out_lat, const void* w_uv,
                        const void* w_o, const void* gate, int64_t n_rows, void* y, void* workspace,
                        size_t workspace_bytes, void* stream) {
  return out_project_impl(dims, dtype, out_lat, false, w_uv, w_o, gate, n_rows, y, workspace, workspace_bytes,
                          stream);
}

int32_t mla_out_project_bf16(const mla_dims* dims, const void* out_lat, const void* w_uv, const void* w_o,
                             const void* gate, int64_t n_rows, void* y, void* workspace, size_t workspace_bytes,
                             void* stream) {
  return out_project_impl(dims, MLA_BF16, out_lat, true, w_uv, w_o, gate, n_rows, y, workspace, workspace_bytes,
                          stream);
}

int32_t mla_linear(int32_t dtype, const void* x, const void* w, int64_t m, int64_t n, int64_t k,
                   uint32_t flags, void* y, void* stream) {
  if (!dtype_ok(dtype)) return MLA_ERR_DTYPE;
  if (flags & ~(uint32_t)(MLA_LINEAR_SIGMOID | MLA_LINEAR_W_KN)) return MLA_ERR_MODE;
  if (m < 0 || n < 0 || k < 0) return MLA_ERR_SHAPE;
  if (m == 0 || n == 0) return MLA_OK;
  if (!x || !w || !y) return MLA_ERR_NULL;
  int st = check_align(dtype, {x, w, y});
  if (st) return st;
  cudaStream_t s = as_stream(stream);
  const bool kn = (flags & MLA_LINEAR_W_KN) != 0;
  const int sig = (flags & MLA_LINEAR_SIGMOID) ? 1 : 0;
  if (dtype == MLA_BF16 && !kn && tc_linear_supported(m, n, k))
    return tc_linear(x, w, m, n, k, sig, y, s);
  GemmArgs g{};
  g.A = x; g.sa_b = 0; g.sa_m = k; g.sa_k = 1;
  g.B = w; g.sb_b = 0; g.sb_n = kn ? 1 : k; g.sb_k = kn ? n : 1;
  g.C = y; g.sc_b = 0; g.sc_m = n; g.sc_n = 1;
  g.M = m; g.N = n; g.K = k; g.batch = 1; g.sigmoid = sig;
  return gemm_generic(g, dtype, dtype, dtype, dtype, s);
}

// ---------------------------------------------------------------------------------------------
// input projections fused with the append
// ---------------------------------------------------------------------------------------------
static int check_project_sizes(const mla_dims* dims, int32_t dtype, int32_t q_rank, int64_t n_rows) {
  int st = check_dims(dims);
  if (st) return st;
  if (!dtype_ok(dtype)) return MLA_ERR_DTYPE;
  if (q_rank <= 0 || n_rows < 0 || dims->qk_nope <= 0 || dims->d_model <= 0) return MLA_ERR_SHAPE;
  if (n_rows > 0x7fffffffLL) return MLA_ERR_SHAPE;
  return MLA_OK;
}

struct ProjectLayout {
  size_t c_q, q_r, kv, partial, total;   // byte offsets in the workspace
};

static ProjectLayout project_layout(const mla_dims* d, int32_t dtype, int64_t q_rank, int64_t n_rows) {
  ProjectLayout L{};
  const size_t es = dtype_bytes(dtype);
  L.c_q = 0;
  L.q_r = L.c_q + round_up((size_t)n_rows * q_rank * es, 256);
  L.kv = L.q_r + round_up((size_t)n_rows * d->n_heads * d->rope_dim * sizeof(float), 256);
  L.partial = L.kv + round_up((size_t)n_rows * (d->kv_lora_rank + d->rope_dim) * sizeof(float), 256);
  L.total = L.partial;
  if (dtype == MLA_BF16 && tc_project_supported(*d, q_rank, n_rows))
    L.total += tc_project_partial_bytes(*d, q_rank, n_rows);
  return L;
}

static int project_generic(const mla_dims* d, int32_t dtype, int64_t q_rank, const void* x, const void* w_cq,
                           const void* w_qc, const void* w_qr, const void* w_dkv, int64_t n_rows, void* c_q,
                           void* q_nope, float* q_r, float* kv, cudaStream_t s) {
  const int64_t H = d->n_heads, n = d->qk_nope, dr = d->rope_dim, W = d->kv_lora_rank + dr, D = d->d_model;
  // out[t, o] = sum_k in[t, k] w[o, k]
  auto linear = [&](const void* in, int32_t in_dt, int64_t k, const void* w, int64_t rows, void* out,
                    int32_t out_dt) {
    GemmArgs g{};
    g.A = in;  g.sa_b = 0; g.sa_m = k; g.sa_k = 1;
    g.B = w;   g.sb_b = 0; g.sb_n = k; g.sb_k = 1;
    g.C = out; g.sc_b = 0; g.sc_m = rows; g.sc_n = 1;
    g.M = n_rows; g.N = rows; g.K = k; g.batch = 1;
    return gemm_generic(g, in_dt, dtype, out_dt, dtype, s);
  };
  int st = linear(x, dtype, D, w_dkv, W, kv, MLA_F32);
  if (st) return st;
  if ((st = linear(x, dtype, D, w_cq, q_rank, c_q, dtype))) return st;
  if ((st = linear(c_q, dtype, q_rank, w_qc, H * n, q_nope, dtype))) return st;
  if (dr > 0) st = linear(c_q, dtype, q_rank, w_qr, H * dr, q_r, MLA_F32);
  return st;
}

int32_t mla_project_workspace_size(const mla_dims* dims, int32_t dtype, int32_t q_rank, int64_t n_rows,
                                   size_t* bytes) {
  if (!bytes) return MLA_ERR_NULL;
  int st = check_project_sizes(dims, dtype, q_rank, n_rows);
  if (st) return st;
  *bytes = project_layout(dims, dtype, q_rank, n_rows).total;
  return MLA_OK;
}

int32_t mla_project_inputs(const mla_dims* dims, int32_t dtype, int32_t q_rank, const void* x, const void* w_cq,
                           const void* w_qc, const void* w_qr, const void* w_dkv, int64_t n_rows,
                           const int32_t* positions, void* q_nope, void* q_pe, void* cache, int64_t cache_rows,
                           const int64_t* row_idx, uint32_t flags, float eps, float rope_theta, void* workspace,
                           size_t workspace_bytes, void* stream) {
  int st = check_project_sizes(dims, dtype, q_rank, n_rows);
  if (st) return st;
  if (flags & ~(uint32_t)(MLA_APPEND_NORM | MLA_APPEND_ROPE)) return MLA_ERR_MODE;
  if (cache_rows < 0) return MLA_ERR_SHAPE;
  if (n_rows == 0) return MLA_OK;
  const int64_t dr = dims->rope_dim;
  if (!x || !w_cq || !w_qc || !w_dkv || !q_nope || !cache || !row_idx) return MLA_ERR_NULL;
  if (dr > 0 && (!w_qr || !q_pe)) return MLA_ERR_NULL;
  if ((flags & MLA_APPEND_ROPE) && dr > 0) {
    if (!positions) return MLA_ERR_NULL;
    if (dr % 2) return MLA_ERR_SHAPE;
    if (!(rope_theta > 0.f)) return MLA_ERR_SHAPE;
  }
  if ((flags & MLA_APPEND_NORM) && !(eps >= 0.f)) return MLA_ERR_SHAPE;
  if ((st = check_align(dtype, {x, w_cq, w_qc, w_qr, w_dkv, q_nope, q_pe, cache}))) return st;
  const ProjectLayout L = project_layout(dims, dtype, q_rank, n_rows);
  if (!workspace || workspace_bytes < L.total) return MLA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return MLA_ERR_ALIGN;
  char* ws = static_cast<char*>(workspace);
  void* c_q = ws + L.c_q;
  float* q_r = reinterpret_cast<float*>(ws + L.q_r);
  float* kv = reinterpret_cast<float*>(ws + L.kv);
  cudaStream_t s = as_stream(stream);
  const bool rotate = (flags & MLA_APPEND_ROPE) != 0;
  const int64_t W = dims->kv_lora_rank + dr;
  // the rotary-query product may come back as K-split partials, which the rotation adds in order
  ProjectParts parts{q_r, 1, 0};
  if (dtype == MLA_BF16 && tc_project_supported(*dims, q_rank, n_rows)) {
    // The KV branch (down-projection, its split-K sum, the append) does not depend on the query chain:
    // it runs on the library's side stream of this device, forked from and joined back to the caller's
    // stream, so that its short kernels overlap the query products.
    // (Without a side stream, e.g. when none can be made, the branch runs on the caller's stream.)
    SideStream* side = side_stream();
    std::unique_lock<std::mutex> lock;
    cudaStream_t s_kv = s;
    if (side) {
      lock = std::unique_lock<std::mutex>(side->m);
      if (cudaEventRecord(side->fork, s) != cudaSuccess || cudaStreamWaitEvent(side->s, side->fork, 0) != cudaSuccess)
        return MLA_ERR_CUDA;
      s_kv = side->s;
    }
    st = tc_project(*dims, q_rank, x, w_cq, w_qc, w_qr, w_dkv, n_rows, c_q, q_nope, q_r, kv, ws + L.partial, s,
                    &parts, s_kv);
    if (!st)
      st = append_latent_strided(*dims, dtype, cache, cache_rows, row_idx, kv, W, kv + dims->kv_lora_rank, W,
                                 positions, n_rows, flags, eps, rope_theta, s_kv);
    // join (also after an error, so that the caller's stream never runs ahead of the side stream's work),
    // before the rotation: a wait between two kernels ends their programmatic overlap, and the rotation
    // gains less from it than the caller's next kernel (which prefetches its weights during the
    // rotation's tail)
    if (side && (cudaEventRecord(side->join, side->s) != cudaSuccess || cudaStreamWaitEvent(s, side->join, 0) != cudaSuccess))
      return MLA_ERR_CUDA;
    if (!st && dr > 0)
      st = rope_rows_launch(dtype, parts.qr, q_pe, positions, n_rows, dims->n_heads, (int)dr, rotate, rope_theta, s,
                            parts.qr_parts, parts.qr_stride);
    return st;
  }
  st = project_generic(dims, dtype, q_rank, x, w_cq, w_qc, w_qr, w_dkv, n_rows, c_q, q_nope, q_r, kv, s);
  if (st) return st;
  if (dr > 0 && (st = rope_rows_launch(dtype, parts.qr, q_pe, positions, n_rows, dims->n_heads, (int)dr, rotate,
                                       rope_theta, s, parts.qr_parts, parts.qr_stride)))
    return st;
  return append_latent_strided(*dims, dtype, cache, cache_rows, row_idx, kv, W, kv + dims->kv_lora_rank, W, positions,
                               n_rows, flags, eps, rope_theta, s);
}

// ---------------------------------------------------------------------------------------------
// one decode step: project -> append -> absorb -> decode -> value/output projection
// ---------------------------------------------------------------------------------------------
struct StepLayout {
  // byte offsets in the workspace
  size_t x_in, y_out, cu, rows, pos;     // staging of the host buffers (MLA_IO_HOST)
  size_t q_nope, q_pe, q_abs, out_lat;   // the step's intermediates
  size_t scratch;                        // shared by the projection, the decode and the output projection
  size_t total;
  size_t proj_bytes, dec_bytes, out_bytes;
};

static int step_layout(const mla_dims* d, int32_t dtype, int32_t q_rank, int32_t batch, int64_t max_seqlen,
                       int64_t total_rows, StepLayout* L) {
  const size_t es = dtype_bytes(dtype);
  const size_t n = (size_t)batch, H = d->n_heads, dc = d->kv_lora_rank, dr = d->rope_dim;
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o += round_up(bytes, 256); return at; };
  L->x_in = take(n * d->d_model * es);
  L->y_out = take(n * d->d_model * es);
  L->cu = take((n + 1) * sizeof(int32_t));
  L->rows = take(n * sizeof(int64_t));
  L->pos = take(n * sizeof(int32_t));
  L->q_nope = take(n * H * d->qk_nope * es);
  L->q_pe = take(n * H * dr * es);
  L->q_abs = take(n * H * (dc + dr) * es);
  L->out_lat = take(n * H * dc * sizeof(float));
  L->scratch = o;
  int st = mla_project_workspace_size(d, dtype, q_rank, batch, &L->proj_bytes);
  if (st) return st;
  if ((st = mla_decode_workspace_size(d, dtype, batch, 1, max_seqlen, total_rows, MLA_DECODE_CAUSAL,
                                      &L->dec_bytes)))
    return st;
  if ((st = mla_out_project_workspace_size(d, dtype, batch, &L->out_bytes))) return st;
  L->total = o + round_up(std::max(L->proj_bytes, std::max(L->dec_bytes, L->out_bytes)), 256);
  return MLA_OK;
}

int32_t mla_decode_step_workspace_size(const mla_dims* dims, int32_t dtype, int32_t q_rank, int32_t batch,
                                       int64_t max_seqlen, int64_t total_rows, size_t* bytes) {
  if (!bytes) return MLA_ERR_NULL;
  int st = check_project_sizes(dims, dtype, q_rank, batch);
  if (st) return st;
  if ((st = check_decode_sizes(dims, dtype, batch, 1, max_seqlen, total_rows, MLA_DECODE_CAUSAL))) return st;
  StepLayout L{};
  if ((st = step_layout(dims, dtype, q_rank, batch, max_seqlen, total_rows, &L))) return st;
  *bytes = L.total;
  return MLA_OK;
}

int32_t mla_decode_step(const mla_dims* dims, int32_t dtype, int32_t q_rank, const mla_step_weights* w,
                        const void* x, void* cache, const int32_t* cu_seqlens, int32_t batch, int64_t max_seqlen,
                        int64_t total_rows, const int64_t* row_idx, const int32_t* positions,
                        uint32_t append_flags, float eps, float rope_theta, void* y, int32_t io, void* workspace,
                        size_t workspace_bytes, void* stream) {
  int st = check_project_sizes(dims, dtype, q_rank, batch);
  if (st) return st;
  if ((st = check_decode_sizes(dims, dtype, batch, 1, max_seqlen, total_rows, MLA_DECODE_CAUSAL))) return st;
  if (io != MLA_IO_DEVICE && io != MLA_IO_HOST) return MLA_ERR_MODE;
  if (batch == 0) return MLA_OK;
  if (!w || !x || !cache || !cu_seqlens || !row_idx || !y) return MLA_ERR_NULL;
  if (!w->w_cq || !w->w_qc || !w->w_dkv || !w->w_uk || !w->w_uv || !w->w_o) return MLA_ERR_NULL;
  if (dims->rope_dim > 0 && !w->w_qr) return MLA_ERR_NULL;
  if (dims->v_head <= 0) return MLA_ERR_SHAPE;
  StepLayout L{};
  if ((st = step_layout(dims, dtype, q_rank, batch, max_seqlen, total_rows, &L))) return st;
  if (!workspace || workspace_bytes < L.total) return MLA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return MLA_ERR_ALIGN;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t s = as_stream(stream);
  const size_t es = dtype_bytes(dtype);
  const size_t x_bytes = (size_t)batch * dims->d_model * es;
  if (io == MLA_IO_HOST) {
    // the step's inputs into the staging area; with pinned host memory these copies (and the output's)
    // are asynchronous and the call returns once everything is enqueued on `stream`
    const bool need_pos = (append_flags & MLA_APPEND_ROPE) && dims->rope_dim > 0;
    if (need_pos && !positions) return MLA_ERR_NULL;
    if (cudaMemcpyAsync(ws + L.x_in, x, x_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) return MLA_ERR_CUDA;
    // the small index arrays travel in one kernel's launch parameters (read now); beyond that kernel's
    // capacity, or while the stream is being captured into a graph (whose replays must read the host
    // buffers again, as a captured copy does), by copies of their own
    cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &capture) != cudaSuccess) return MLA_ERR_CUDA;
    st = capture != cudaStreamCaptureStatusNone
             ? MLA_ERR_UNSUPPORTED
             : put_step_indices(cu_seqlens, row_idx, need_pos ? positions : nullptr, batch,
                                reinterpret_cast<int32_t*>(ws + L.cu), reinterpret_cast<int64_t*>(ws + L.rows),
                                reinterpret_cast<int32_t*>(ws + L.pos), s);
    if (st == MLA_ERR_UNSUPPORTED) {
      if (cudaMemcpyAsync(ws + L.cu, cu_seqlens, (size_t)(batch + 1) * sizeof(int32_t), cudaMemcpyHostToDevice,
                          s) != cudaSuccess ||
          cudaMemcpyAsync(ws + L.rows, row_idx, (size_t)batch * sizeof(int64_t), cudaMemcpyHostToDevice, s) !=
              cudaSuccess ||
          (need_pos && cudaMemcpyAsync(ws + L.pos, positions, (size_t)batch * sizeof(int32_t),
                                       cudaMemcpyHostToDevice, s) != cudaSuccess))
        return MLA_ERR_CUDA;
    } else if (st) {
      return st;
    }
    x = ws + L.x_in;
    cu_seqlens = reinterpret_cast<const int32_t*>(ws + L.cu);
    row_idx = reinterpret_cast<const int64_t*>(ws + L.rows);
    if (need_pos) positions = reinterpret_cast<const int32_t*>(ws + L.pos);
  }
  void* q_nope = ws + L.q_nope;
  void* q_pe = ws + L.q_pe;
  void* q_abs = ws + L.q_abs;
  float* out_lat = reinterpret_cast<float*>(ws + L.out_lat);
  void* scratch = ws + L.scratch;
  void* y_dev = io == MLA_IO_HOST ? static_cast<void*>(ws + L.y_out) : y;
  if ((st = mla_project_inputs(dims, dtype, q_rank, x, w->w_cq, w->w_qc, w->w_qr, w->w_dkv, batch, positions,
                               q_nope, q_pe, cache, total_rows, row_idx, append_flags, eps, rope_theta, scratch,
                               L.proj_bytes, stream)))
    return st;
  if ((st = mla_absorb_weights(dims, dtype, MLA_ABSORB_QUERY, q_nope, q_pe, w->w_uk, batch, q_abs, stream)))
    return st;
  // on the tensor-core route the decode writes out_lat in bf16, the W_UV operand, directly
  st = dtype == MLA_BF16 ? mla_decode_absorbed(dims, dtype, q_abs, cache, cu_seqlens, batch, 1, max_seqlen, total_rows,
                                               MLA_DECODE_CAUSAL | MLA_DECODE_OUT_BF16, out_lat, nullptr, scratch,
                                               L.dec_bytes, stream)
                         : MLA_ERR_UNSUPPORTED;
  if (st == MLA_OK) {
    st = mla_out_project_bf16(dims, out_lat, w->w_uv, w->w_o, nullptr, batch, y_dev, scratch, L.out_bytes, stream);
  } else if (st == MLA_ERR_UNSUPPORTED) {
    if ((st = mla_decode_absorbed(dims, dtype, q_abs, cache, cu_seqlens, batch, 1, max_seqlen, total_rows,
                                  MLA_DECODE_CAUSAL, out_lat, nullptr, scratch, L.dec_bytes, stream)))
      return st;
    st = mla_out_project(dims, dtype, out_lat, w->w_uv, w->w_o, nullptr, batch, y_dev, scratch, L.out_bytes, stream);
  }
  if (st) return st;
  if (io == MLA_IO_HOST && cudaMemcpyAsync(y, y_dev, x_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}

int32_t mla_prefill_attention(int32_t dtype, const void* q, const void* k, const void* v, const void* gate,
                              int32_t batch, int32_t seq, int32_t n_heads, int32_t head_dim, float scale,
                              uint32_t flags, void* out, void* stream) {
  if (!dtype_ok(dtype)) return MLA_ERR_DTYPE;
  if (flags & ~(uint32_t)MLA_DECODE_CAUSAL) return MLA_ERR_MODE;
  if (batch < 0 || seq < 0 || n_heads <= 0 || head_dim <= 0) return MLA_ERR_SHAPE;
  if (!(scale >= 0.f) || isinf(scale)) return MLA_ERR_SHAPE;
  if (batch == 0 || seq == 0) return MLA_OK;
  if (!q || !k || !v || !out) return MLA_ERR_NULL;
  if (dtype != MLA_BF16 || !tc_prefill_supported(batch, seq, n_heads, head_dim)) return MLA_ERR_UNSUPPORTED;
  int st = check_align(dtype, {q, k, v, gate, out});
  if (st) return st;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)head_dim);
  return tc_prefill_launch(q, k, v, gate, batch, seq, n_heads, sc, (flags & MLA_DECODE_CAUSAL) != 0, out,
                           as_stream(stream));
}

int32_t mla_lse_merge(const mla_dims* dims, int32_t n_parts, const float* const* out_lat_parts,
                      const float* const* lse_parts, int64_t row_begin, int64_t n_rows, float* out_lat, float* lse,
                      void* stream) {
  int st = check_dims(dims);
  if (st) return st;
  if (n_parts < 1 || n_parts > MLA_MERGE_MAX_PARTS || row_begin < 0 || n_rows < 0) return MLA_ERR_SHAPE;
  if (n_rows == 0) return MLA_OK;
  if (!out_lat_parts || !lse_parts || !out_lat) return MLA_ERR_NULL;
  for (int r = 0; r < n_parts; ++r) {
    if (!out_lat_parts[r] || !lse_parts[r]) return MLA_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(out_lat_parts[r]) & 15u) return MLA_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(lse_parts[r]) & 3u) return MLA_ERR_ALIGN;
  }
  if ((reinterpret_cast<uintptr_t>(out_lat) & 15u) || (reinterpret_cast<uintptr_t>(lse) & 3u)) return MLA_ERR_ALIGN;
  return lse_merge_launch(n_parts, out_lat_parts, lse_parts, row_begin, n_rows, dims->n_heads, dims->kv_lora_rank,
                          out_lat, lse, as_stream(stream));
}

int32_t mla_check_status(void* stream, int32_t* device_status) {
  if (!device_status) return MLA_ERR_NULL;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return MLA_ERR_CUDA;
  int* p = device_status_ptr();
  if (!p) return MLA_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return MLA_ERR_CUDA;
  *device_status = v;
  return MLA_OK;
}

int32_t mla_set_decode_clusters(int32_t n) {
  if (n < 0) return MLA_ERR_SHAPE;
  set_decode_clusters(n);
  return MLA_OK;
}

int64_t mla_launch_count(void) { return (int64_t)launch_count(); }

int32_t mla_set_wait_limit(int64_t limit_ns) {
  if (limit_ns < 0) return MLA_ERR_SHAPE;
  set_wait_limit((long long)limit_ns);
  return MLA_OK;
}

int32_t mla_wait_selftest(void* stream) { return wait_selftest_launch(as_stream(stream)); }

}  // extern "C"
