// mla_api.cu -- the C ABI declared in include/mla.h: host-side validation and kernel dispatch.
#include <math.h>
#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "tc.cuh"

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

int32_t mla_abi_version(void) { return 1; }

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
  if (flags & ~(uint32_t)MLA_DECODE_CAUSAL) return MLA_ERR_MODE;
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
  int st = check_decode_sizes(dims, dtype, batch, n_q, max_seqlen, total_rows, flags);
  if (st) return st;
  DecodeArgs a = make_decode_args(dims, batch, n_q, max_seqlen, total_rows, flags);
  if (dtype == MLA_BF16 && tc_decode_supported(a))
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
  if (dtype == MLA_BF16 && tc_decode_supported(a)) {
    if (workspace_bytes < tc_decode_workspace(a) || !workspace) return MLA_ERR_WORKSPACE;
    return tc_decode_launch(a, s);
  }
  if (workspace_bytes < decode_generic_workspace(a)) return MLA_ERR_WORKSPACE;
  return decode_generic_launch(a, dtype, s);
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

int32_t mla_out_project(const mla_dims* dims, int32_t dtype, const float* out_lat, const void* w_uv,
                        const void* w_o, const void* gate, int64_t n_rows, void* y, void* workspace,
                        size_t workspace_bytes, void* stream) {
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
    return tc_out_project(*dims, out_lat, w_uv, w_o, gate, n_rows, y, workspace, workspace_bytes, s);
  // stage 1: v[t, h, i] = gate * sum_j out_lat[t, h, j] W_UV[h, i, j]; batch = h, M = t, N = i
  GemmArgs g{};
  g.A = out_lat; g.sa_b = dc; g.sa_m = H * dc; g.sa_k = 1;
  g.B = w_uv;    g.sb_b = dv * dc; g.sb_n = dc; g.sb_k = 1;
  g.C = v;       g.sc_b = dv; g.sc_m = H * dv; g.sc_n = 1;
  g.G = gate;    g.sg_b = dv; g.sg_m = H * dv; g.sg_n = 1;
  g.M = n_rows; g.N = dv; g.K = dc; g.batch = H;
  if ((st = gemm_generic(g, MLA_F32, dtype, dtype, dtype, s))) return st;
  // stage 2: y[t, d] = sum_k v[t, k] W_O[d, k]
  GemmArgs o{};
  o.A = v;   o.sa_b = 0; o.sa_m = H * dv; o.sa_k = 1;
  o.B = w_o; o.sb_b = 0; o.sb_n = H * dv; o.sb_k = 1;
  o.C = y;   o.sc_b = 0; o.sc_m = D; o.sc_n = 1;
  o.M = n_rows; o.N = D; o.K = H * dv; o.batch = 1;
  return gemm_generic(o, dtype, dtype, dtype, dtype, s);
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
