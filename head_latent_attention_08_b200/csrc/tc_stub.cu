// tc_stub.cu -- placeholder: tensor-core paths not yet enabled; every request takes the CUDA-core path.
#include "tc.cuh"

namespace mla {
bool tc_absorb_supported(const mla_dims&, int64_t) { return false; }
int tc_absorb_query(const mla_dims&, const void*, const void*, const void*, int64_t, void*, cudaStream_t) { return MLA_ERR_UNSUPPORTED; }
bool tc_decode_supported(const DecodeArgs&) { return false; }
size_t tc_decode_workspace(const DecodeArgs&) { return 0; }
int tc_decode_launch(const DecodeArgs&, cudaStream_t) { return MLA_ERR_UNSUPPORTED; }
bool tc_out_project_supported(const mla_dims&, int64_t) { return false; }
size_t tc_out_project_extra_workspace(const mla_dims&, int64_t) { return 0; }
int tc_out_project(const mla_dims&, const float*, const void*, const void*, const void*, int64_t, void*, void*, size_t, cudaStream_t) { return MLA_ERR_UNSUPPORTED; }
bool tc_linear_supported(int64_t, int64_t, int64_t) { return false; }
int tc_linear(const void*, const void*, int64_t, int64_t, int64_t, int, void*, cudaStream_t) { return MLA_ERR_UNSUPPORTED; }
}  // namespace mla
