// tc.cuh -- entry points of the tensor-core (tcgen05 / TMA / TMEM) kernels for sm_100a.
#pragma once

#include "common.cuh"

namespace mla {

// query absorption q_abs = W_UK^T q_nope per head (bf16 in, fp32 accumulate, bf16 out)
bool tc_absorb_supported(const mla_dims& d, int64_t n_rows);
int tc_absorb_query(const mla_dims& d, const void* q_nope, const void* q_pe, const void* w_uk,
                    int64_t n_rows, void* q_abs, cudaStream_t s);

// fused split-KV absorbed decode
bool tc_decode_supported(const DecodeArgs& a);
size_t tc_decode_workspace(const DecodeArgs& a);
int tc_decode_launch(const DecodeArgs& a, cudaStream_t s);
void set_decode_clusters(int n);   // 0 = one cluster per SM pair

// value + output projection
bool tc_out_project_supported(const mla_dims& d, int64_t n_rows);
size_t tc_out_project_extra_workspace(const mla_dims& d, int64_t n_rows);
int tc_out_project(const mla_dims& d, const void* out_lat, bool lat_bf16, const void* w_uv, const void* w_o,
                   const void* gate, int64_t n_rows, void* y, void* workspace, size_t ws_bytes, cudaStream_t s);

// input projections of new tokens (bf16 in, fp32 accumulate): c_q = x W_cq^T and q_nope = c_q W_qc^T
// in bf16, q_r = c_q W_qr^T and kv = x W_dkv^T in fp32; partial = split-K scratch of
// tc_project_partial_bytes() bytes
// The KV and rotary-query products come back as `parts` fp32 arrays `stride` floats apart (their
// K-split partials, to be added in order; one array when the product was not split).
struct ProjectParts {
  const float* qr;     // the rotary query product q_r, or its first K-split partial
  int qr_parts;        // partials to add in order (1: q_r itself)
  int64_t qr_stride;   // floats between partials
};
bool tc_project_supported(const mla_dims& d, int64_t q_rank, int64_t n_rows);
size_t tc_project_partial_bytes(const mla_dims& d, int64_t q_rank, int64_t n_rows);
// the KV down-projection runs on s_kv (may be s), the query chain on s
int tc_project(const mla_dims& d, int64_t q_rank, const void* x, const void* w_cq, const void* w_qc,
               const void* w_qr, const void* w_dkv, int64_t n_rows, void* c_q, void* q_nope, float* q_r,
               float* kv, void* partial, cudaStream_t s, ProjectParts* parts, cudaStream_t s_kv);
// attention of un-absorbed heads over whole prompts (bf16, head width 128): q, k, v, out and the
// optional gate are [B*S, H*128]; out = softmax(scale q k^T, causal or full) v (times the gate)
bool tc_prefill_supported(int64_t B, int64_t S, int64_t H, int64_t D);
int tc_prefill_launch(const void* q, const void* k, const void* v, const void* gate, int64_t B, int64_t S, int64_t H,
                      float scale, bool causal, void* out, cudaStream_t s);
// dense linear Y = X W^T
bool tc_linear_supported(int64_t m, int64_t n, int64_t k);
int tc_linear(const void* x, const void* w, int64_t m, int64_t n, int64_t k, int sigmoid, void* y,
              cudaStream_t s);

// one CTA waiting, through the bounded wait of the tensor-core kernels, on a barrier nothing completes
int wait_selftest_launch(cudaStream_t s);

}  // namespace mla
