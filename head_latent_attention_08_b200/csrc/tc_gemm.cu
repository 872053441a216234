// tc_gemm.cu -- tensor-core GEMM for sm_100a (TMA -> shared memory -> tcgen05.mma -> TMEM) and the
// three products of the absorbed form that run on it:
//   * query absorption  q_abs[t,h,:d_c] = W_UK[h]^T q_nope[t,h]   (per head: M = d_c, N = tokens)
//   * value projection  v[t,h] = gate * (W_UV[h] out_lat[t,h])      (per head: M = v_head, N = tokens)
//   * output projection y[t] = W_O v[t]                            (M = d_model, N = tokens, split-K)
//   * dense linear      Y = X W^T                                  (M = out features, N = tokens)
//
// Shape of one CTA: D[128 x BN] (fp32, TMEM) = A[128 x K] . B[BN x K]^T with A the weight tile and B
// the token tile, both bf16 in 128-byte-swizzled shared memory, fed by TMA through a ring of stages.
// One thread issues the TMA loads, one thread issues the MMAs (4 x K16 per 64-wide K chunk), and the
// four warps drain TMEM in the epilogue (warp w owns accumulator rows 32w..32w+31). The result is
// stored transposed, out[t][m]: consecutive lanes write consecutive addresses. Weights wider than one
// wave of tiles are split along K; the fp32 partials are summed in a fixed order by a second kernel.
// Products with more tiles than SMs and long K (the dense linears of a prefill) run on a persistent
// form instead: one CTA per SM walks several tiles, with two TMEM accumulators so that one tile's
// epilogue (four dedicated warps) overlaps the next tile's loads and MMAs.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "sm100.cuh"
#include "tc.cuh"

namespace mla {

using namespace sm100;

// ---------------------------------------------------------------------------------------------
// host: tensor maps
// ---------------------------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      (void)cudaGetLastError();
  });
  return fn;
}

static bool encode_tmap(CUtensorMap* map, CUtensorMapDataType type, void* base, int rank, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  CUresult r = fn(map, type, (cuuint32_t)rank, base, d, st, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_bf16(CUtensorMap* map, void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes) {
  return encode_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes, box,
                     swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

bool encode_tmap_u8(CUtensorMap* map, void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                    const uint32_t* box, int swizzle_bytes) {
  return encode_tmap(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, rank, dims, strides_bytes, box,
                     swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

// ---------------------------------------------------------------------------------------------
// the GEMM kernel
// ---------------------------------------------------------------------------------------------
struct TcGemmParams {
  int M, N, K;
  int m_tiles;       // 128-row tiles of the weight
  int n_tiles;       // BN-wide token tiles
  int k_chunks;      // 64-wide K chunks per split
  int n_splits;
  int batch;
  void* out; int64_t out_sb, out_st; int out_f32;
  const __nv_bfloat16* gate; int64_t gate_sb, gate_st;
  float* partial;    // [split][batch][N][M] when n_splits > 1
  int sigmoid;
  int stages;        // depth of the shared-memory ring (<= GemmCfg::STAGES; sized to the K chunks)
  // optional tail: out[bz][t][tail_off + c] = tail[bz * tail_sb + t * tail_st + c], c < tail_cols
  // (copied by the m-tile-0, split-0 CTA of each token tile; bf16 output only, 16-byte rows)
  const __nv_bfloat16* tail; int64_t tail_sb, tail_st, tail_off; int tail_cols;
  int* status;
  unsigned long long wait_ns;
};

constexpr int GEMM_PRODUCERS = 3;   // warps issuing the TMA loads (0, 2 and 3; warp 1 issues the MMAs)

template <int BN>
struct GemmCfg {
  static constexpr int A_BYTES = 128 * 64 * 2;
  static constexpr int B_BYTES = BN * 64 * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES_FIT = (192 * 1024) / STAGE;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int SMEM = STAGES * STAGE + 1024 + 256;
  static constexpr uint32_t TMEM_COLS = BN < 32 ? 32 : BN;
};

template <int BN, bool A_MN>
__global__ void __launch_bounds__(128, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
                   TcGemmParams p) {
  using Cfg = GemmCfg<BN>;
  const int STAGES = p.stages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::STAGE);
  uint64_t* empty = full + STAGES;
  uint64_t* done = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_load = abort_flag + 1;   // [STAGES]: the last K chunk loaded into each stage

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128;
  const int split = blockIdx.y / p.n_tiles, n0 = (blockIdx.y % p.n_tiles) * BN;
  const int bz = blockIdx.z;
  const int total_chunks = (p.K + 63) / 64;
  const int kc0 = split * p.k_chunks;
  const int nk = max(0, min(kc0 + p.k_chunks, total_chunks) - kc0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) last_load[s] = -1;
    fence_mbar_init();
    prefetch_tmap(&ta);
    prefetch_tmap(&tb);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Producers in use: never more than the ring has stages. A producer waits for the release of its
  // chunk's stage by parity, which is only sound while that stage's previous round has been loaded:
  // with P producers taking every P-th chunk, that holds when STAGES >= P.
  const int nprod = min(GEMM_PRODUCERS, STAGES);
  const bool producer = warp != 1 && lane == 0 && (warp == 0 ? 0 : warp - 1) < nprod;
  // the activations (B), the gate and the tail may come from the previous kernel of the stream, and the
  // output may still be read by it: everyone waits for it, the producers after their weight prefetch
  if (!producer) griddep_wait();
  griddep_launch_dependents();
  const uint32_t tmem_d = *tmem_slot;

  if (producer) {
    // TMA producers, lane 0 of warps 0, 2 and 3: producer j loads K chunks j, j + P, j + 2P, ... (an
    // SM moves more bytes with bulk copies issued from several warps than from one thread). Chunk i
    // goes to stage i % STAGES, whose previous round the MMAs must have released first.
    const int j = warp == 0 ? 0 : warp - 1;
    auto load_a = [&](int i, int s) {
      uint8_t* a_dst = smem + s * Cfg::STAGE;
      const int kx = (kc0 + i) * 64;
      if (A_MN) {
        tma_load_3d(a_dst, &ta, &full[s], m0, kx, bz);
        tma_load_3d(a_dst + 8192, &ta, &full[s], m0 + 64, kx, bz);
      } else {
        tma_load_3d(a_dst, &ta, &full[s], kx, m0, bz);
      }
    };
    // The weights (A) are never written by the library's kernels: the first ring's weight tiles are
    // requested before the wait, so that their latency overlaps the previous kernel's tail.
    const int pre = min(nk, STAGES);
    for (int i = j; i < pre; i += nprod) {
      mbar_arrive_expect_tx(&full[i], Cfg::STAGE);
      load_a(i, i);
      last_load[i] = i;
    }
    griddep_wait();
    for (int i = j; i < nk; i += nprod) {
      const int s = i % STAGES;
      if (i >= STAGES) {      // (a prefetched stage always gets its B tile, so that its barrier completes)
        if (!mbar_wait(&empty[s], (uint32_t)(((i / STAGES) - 1) & 1), p.wait_ns, p.status)) {
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        mbar_arrive_expect_tx(&full[s], Cfg::STAGE);
        load_a(i, s);
        last_load[s] = i;
      }
      tma_load_3d(smem + s * Cfg::STAGE + Cfg::A_BYTES, &tb, &full[s], (kc0 + i) * 64, n0, bz);
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(128, BN, A_MN, false);
    int s = 0, ph = 0;
    for (int i = 0; i < nk; ++i) {
      if (!mbar_wait(&full[s], (uint32_t)ph, p.wait_ns, p.status)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t a_base = smem_u32(smem + s * Cfg::STAGE);
      const uint32_t b_base = a_base + Cfg::A_BYTES;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = A_MN ? smem_desc_sw128(a_base + kk * 2048, 8192, 1024)
                                 : smem_desc_sw128(a_base + kk * 32, 16, 1024);
        const uint64_t bd = smem_desc_sw128(b_base + kk * 32, 16, 1024);
        mma_bf16_ss(tmem_d, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(&empty[s]);
      if (++s == STAGES) { s = 0; ph ^= 1; }
    }
    mma_commit(done);
  }
  __syncwarp();

  // epilogue: thread = accumulator row m. The tile goes out through shared memory (the ring is idle
  // once `done` has completed: every load has landed and every MMA has read it), 32 tokens at a time:
  // thread m writes its 32 values to column m of a [32][128] fp32 tile, then the block writes whole
  // 16-byte runs of 4 consecutive outputs of each token row (out[t][m] is contiguous along m).
  const bool ok = mbar_wait(done, 0, p.wait_ns, p.status);
  if (!ok) *abort_flag = 1;
  tc_fence_after();
  const bool write = ok && !*abort_flag;
  float* tile = reinterpret_cast<float*>(smem);          // [32][128]
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    uint32_t r[32];
    tmem_ld32(tmem_d + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, r);
    tmem_wait_ld();
    __syncthreads();                                      // the previous chunk's tile has been read
    if (write) {                                          // (an abandoned CTA may still have loads landing)
#pragma unroll
      for (int j = 0; j < 32; ++j) tile[j * 128 + threadIdx.x] = nk > 0 ? __uint_as_float(r[j]) : 0.f;
    }
    __syncthreads();
    if (write) {
#pragma unroll 2
      for (int q = threadIdx.x; q < 32 * 32; q += 128) {
        const int tl = q >> 5, mq = (q & 31) * 4;
        const int t = n0 + c + tl, m = m0 + mq;
        if (t >= p.N || m >= p.M) continue;
        float4 v = *reinterpret_cast<const float4*>(tile + tl * 128 + mq);
        if (p.n_splits > 1) {
          *reinterpret_cast<float4*>(p.partial + (((int64_t)split * p.batch + bz) * p.N + t) * p.M + m) = v;
          continue;
        }
        if (p.sigmoid) {
          v.x = 1.f / (1.f + expf(-v.x)); v.y = 1.f / (1.f + expf(-v.y));
          v.z = 1.f / (1.f + expf(-v.z)); v.w = 1.f / (1.f + expf(-v.w));
        }
        if (p.gate) {
          const uint2 gv = *reinterpret_cast<const uint2*>(p.gate + bz * p.gate_sb + (int64_t)t * p.gate_st + m);
          const float2 g0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv.x));
          const float2 g1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv.y));
          v.x *= g0.x; v.y *= g0.y; v.z *= g1.x; v.w *= g1.y;
        }
        const int64_t o = bz * p.out_sb + (int64_t)t * p.out_st + m;
        if (p.out_f32) {
          *reinterpret_cast<float4*>(static_cast<float*>(p.out) + o) = v;
        } else {
          __nv_bfloat162 b0 = __floats2bfloat162_rn(v.x, v.y), b1 = __floats2bfloat162_rn(v.z, v.w);
          uint2 w;
          w.x = *reinterpret_cast<uint32_t*>(&b0);
          w.y = *reinterpret_cast<uint32_t*>(&b1);
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.out) + o) = w;
        }
      }
    }
  }
  if (p.tail && write && blockIdx.x == 0 && split == 0) {
    // the tail columns of this CTA's tokens (16-byte chunks; the host checks the alignment)
    const int cpr = p.tail_cols / 8;
    for (int idx = threadIdx.x; idx < BN * cpr; idx += 128) {
      const int t = n0 + idx / cpr, q = idx % cpr;
      if (t >= p.N) break;
      const uint4 v = reinterpret_cast<const uint4*>(p.tail + bz * p.tail_sb + (int64_t)t * p.tail_st)[q];
      reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + bz * p.out_sb + (int64_t)t * p.out_st +
                               p.tail_off)[q] = v;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && *abort_flag) {
    // Abandoned work: neither TMA writes nor MMAs may be left in flight behind the CTA or its tensor
    // memory. Every load issued and the MMA issuer's final commit (made on both of its paths, before
    // the barrier above) complete by themselves; the limit here only bounds the wait. Only the last
    // load of a stage can still be in flight (a later one waited for the MMAs to read the earlier).
    const uint64_t drain_ns = p.wait_ns > 100000000ull ? p.wait_ns : 100000000ull;
    for (int s = 0; s < STAGES; ++s) {
      const int i = last_load[s];
      if (i >= 0) (void)mbar_wait(&full[s], (uint32_t)((i / STAGES) & 1), drain_ns, p.status);
    }
    (void)mbar_wait(done, 0, drain_ns, p.status);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_d, Cfg::TMEM_COLS);
  }
}

// fixed-order sum of split-K partials + epilogue, 4 consecutive outputs per thread (M % 4 == 0; the
// host checks the 16-byte alignment of out and the 8-byte alignment of the gate)
__global__ void splitk_reduce_kernel(const float* __restrict__ partial, int n_splits, int batch, int N, int M,
                                     void* out, int64_t out_sb, int64_t out_st, int out_f32,
                                     const __nv_bfloat16* gate, int64_t gate_sb, int64_t gate_st, int sigmoid) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t per = (int64_t)batch * N * M;
  for (int64_t e = 4 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x); e < per;
       e += 4 * (int64_t)gridDim.x * blockDim.x) {
    float4 v = *reinterpret_cast<const float4*>(partial + e);
#pragma unroll 4
    for (int s = 1; s < n_splits; ++s) {
      const float4 u = *reinterpret_cast<const float4*>(partial + s * per + e);
      v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
    }
    const int m = (int)(e % M);
    const int64_t bt = e / M;
    const int t = (int)(bt % N);
    const int bz = (int)(bt / N);
    if (sigmoid) {
      v.x = 1.f / (1.f + expf(-v.x)); v.y = 1.f / (1.f + expf(-v.y));
      v.z = 1.f / (1.f + expf(-v.z)); v.w = 1.f / (1.f + expf(-v.w));
    }
    if (gate) {
      const uint2 gv = *reinterpret_cast<const uint2*>(gate + bz * gate_sb + (int64_t)t * gate_st + m);
      const float2 g0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv.x));
      const float2 g1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv.y));
      v.x *= g0.x; v.y *= g0.y; v.z *= g1.x; v.w *= g1.y;
    }
    const int64_t o = bz * out_sb + (int64_t)t * out_st + m;
    if (out_f32) {
      *reinterpret_cast<float4*>(static_cast<float*>(out) + o) = v;
    } else {
      __nv_bfloat162 b0 = __floats2bfloat162_rn(v.x, v.y), b1 = __floats2bfloat162_rn(v.z, v.w);
      uint2 w;
      w.x = *reinterpret_cast<uint32_t*>(&b0);
      w.y = *reinterpret_cast<uint32_t*>(&b1);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out) + o) = w;
    }
  }
}

// out_lat fp32 -> bf16 (the tensor-core operand of the value projection)
__global__ void f32_to_bf16_kernel(const float4* __restrict__ src, uint2* __restrict__ dst, int64_t n4) {
  griddep_wait();
  griddep_launch_dependents();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = src[i];
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t*>(&a);
    o.y = *reinterpret_cast<uint32_t*>(&b);
    dst[i] = o;
  }
}

// ---------------------------------------------------------------------------------------------
// persistent form: G CTAs (one per SM at most) walk the units u = c, c + G, c + 2G, ... of the same
// tiling (unit = (batch, split, token tile, 128-row tile), row tile fastest). The shared-memory ring
// runs on across a CTA's units and two TMEM accumulators alternate, so that four epilogue warps drain
// unit u while unit u + 1's tiles load and its MMAs run: a short unit no longer pays its own setup,
// first-load latency and epilogue in series.
//   warps 0, 2, 3: TMA producers (lane 0); warp 1: MMA issuer (lane 0) and TMEM owner;
//   warps 4-7: epilogue (warp 4 + q reads TMEM lanes 32 q .. 32 q + 31 = accumulator rows).
// ---------------------------------------------------------------------------------------------
constexpr int GEMM_P_THREADS = 256;
constexpr int GEMM_P_BAR_BYTES = 256;

template <int BN>
struct GemmPCfg {
  static constexpr int STAGE = GemmCfg<BN>::STAGE;
  static constexpr int FIXED = 1024 + GEMM_P_BAR_BYTES;
  static constexpr int STAGES_FIT = (227 * 1024 - FIXED) / STAGE;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr uint32_t ACC_COLS = GemmCfg<BN>::TMEM_COLS;          // one accumulator
  static constexpr uint32_t TMEM_COLS = 2 * ACC_COLS < 32 ? 32 : 2 * ACC_COLS;
};

struct GemmUnit {
  int m0, n0, split, bz, kc0, nk;
};

__device__ __forceinline__ GemmUnit gemm_unit(const TcGemmParams& p, int64_t u, int BN, int total_chunks) {
  GemmUnit r;
  int64_t x = u;
  const int mt = (int)(x % p.m_tiles);
  x /= p.m_tiles;
  const int nt = (int)(x % p.n_tiles);
  x /= p.n_tiles;
  r.split = (int)(x % p.n_splits);
  r.bz = (int)(x / p.n_splits);
  r.m0 = mt * 128;
  r.n0 = nt * BN;
  r.kc0 = r.split * p.k_chunks;
  r.nk = max(0, min(r.kc0 + p.k_chunks, total_chunks) - r.kc0);
  return r;
}

template <int BN, bool A_MN>
__global__ void __launch_bounds__(GEMM_P_THREADS, 1)
    tc_gemm_persistent_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
                              TcGemmParams p) {
  using Cfg = GemmCfg<BN>;
  using PCfg = GemmPCfg<BN>;
  const int STAGES = p.stages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::STAGE);
  uint64_t* empty = full + 8;
  uint64_t* acc_full = empty + 8;      // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2]
  uint64_t* done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_load = abort_flag + 1;   // [8]: the last chunk (CTA-local count) loaded into each stage

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total_chunks = (p.K + 63) / 64;
  const int64_t U = (int64_t)p.m_tiles * p.n_tiles * p.n_splits * p.batch;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      last_load[s] = -1;
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&ta);
    prefetch_tmap(&tb);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, PCfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // producers in use: no more than the ring has stages (see the one-tile kernel)
  const int nprod = min(GEMM_PRODUCERS, STAGES);
  const bool producer = warp != 1 && warp < 4 && lane == 0 && (warp == 0 ? 0 : warp - 1) < nprod;
  // the activations (B), the gate and the tail may come from the previous kernel of the stream, and the
  // output may still be read by it: everyone waits for it, the producers after their weight prefetch
  if (!producer) griddep_wait();
  griddep_launch_dependents();
  const uint32_t tmem = *tmem_slot;

  auto wait_bar = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity, p.wait_ns, p.status)) return true;
    *abort_flag = 1;
    return false;
  };

  if (producer) {
    // producer j loads the CTA-local chunks g = j, j + P, ... (g counts the chunks of the CTA's units
    // in order); chunk g goes to stage g % STAGES once the MMAs have read its previous round
    const int j = warp == 0 ? 0 : warp - 1;
    auto load_a = [&](const GemmUnit& w, int i, int s) {
      uint8_t* a_dst = smem + s * Cfg::STAGE;
      const int kx = (w.kc0 + i) * 64;
      if (A_MN) {
        tma_load_3d(a_dst, &ta, &full[s], w.m0, kx, w.bz);
        tma_load_3d(a_dst + 8192, &ta, &full[s], w.m0 + 64, kx, w.bz);
      } else {
        tma_load_3d(a_dst, &ta, &full[s], kx, w.m0, w.bz);
      }
    };
    // the weights (A) are never written by the library's kernels: the first ring's weight tiles are
    // requested before the wait, so that their latency overlaps the previous kernel's tail
    int g = 0;
    for (int64_t u = blockIdx.x; u < U && g < STAGES; u += gridDim.x) {
      const GemmUnit w = gemm_unit(p, u, BN, total_chunks);
      for (int i = 0; i < w.nk && g < STAGES; ++i, ++g) {
        if (g % nprod != j) continue;
        mbar_arrive_expect_tx(&full[g], Cfg::STAGE);
        load_a(w, i, g);
        last_load[g] = g;
      }
    }
    griddep_wait();
    g = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < U && ok; u += gridDim.x) {
      const GemmUnit w = gemm_unit(p, u, BN, total_chunks);
      for (int i = 0; i < w.nk; ++i, ++g) {
        if (g % nprod != j) continue;
        const int s = g % STAGES;
        if (g >= STAGES) {    // (a prefetched stage always gets its B tile, so that its barrier completes)
          if (!wait_bar(&empty[s], (uint32_t)(((g / STAGES) - 1) & 1))) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], Cfg::STAGE);
          load_a(w, i, s);
          last_load[s] = g;
        }
        tma_load_3d(smem + s * Cfg::STAGE + Cfg::A_BYTES, &tb, &full[s], (w.kc0 + i) * 64, w.n0, w.bz);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer: unit number ui of this CTA accumulates into TMEM accumulator ui & 1, once the
    // epilogue has drained that accumulator's previous unit
    constexpr uint32_t idesc = idesc_bf16_f32(128, BN, A_MN, false);
    int g = 0, ui = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < U && ok; u += gridDim.x, ++ui) {
      const GemmUnit w = gemm_unit(p, u, BN, total_chunks);
      const int acc = ui & 1;
      if (ui >= 2 && !wait_bar(&acc_empty[acc], (uint32_t)(((ui >> 1) - 1) & 1))) { ok = false; break; }
      tc_fence_after();
      const uint32_t d = tmem + (uint32_t)acc * PCfg::ACC_COLS;
      for (int i = 0; i < w.nk; ++i, ++g) {
        const int s = g % STAGES;
        if (!wait_bar(&full[s], (uint32_t)((g / STAGES) & 1))) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + s * Cfg::STAGE);
        const uint32_t b_base = a_base + Cfg::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = A_MN ? smem_desc_sw128(a_base + kk * 2048, 8192, 1024)
                                   : smem_desc_sw128(a_base + kk * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(b_base + kk * 32, 16, 1024);
          mma_bf16_ss(d, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
      }
      if (!ok) break;
      mma_commit(&acc_full[acc]);
    }
    mma_commit(done);
  } else if (warp >= 4) {
    // ---- epilogue: thread = accumulator row m of unit ui (TMEM lane 32 (warp - 4) + lane); for each
    // token t it stores out[t][m] directly: a warp's store covers 32 consecutive m of one token row
    const int et = threadIdx.x - 128;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    int ui = 0;
    for (int64_t u = blockIdx.x; u < U; u += gridDim.x, ++ui) {
      const GemmUnit w = gemm_unit(p, u, BN, total_chunks);
      const int acc = ui & 1;
      const bool okw = wait_bar(&acc_full[acc], (uint32_t)((ui >> 1) & 1));
      // one decision for the four warps
      if (named_bar_or(1, 128, !okw || *abort_flag)) break;
      tc_fence_after();
      const uint32_t d = tmem + (uint32_t)acc * PCfg::ACC_COLS;
      const int m = w.m0 + et;
      const bool row_ok = m < p.M;
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t r[32];
        tmem_ld32(d + lane_base + (uint32_t)c, r);
        tmem_wait_ld();
        const int nt = min(32, p.N - (w.n0 + c));
        if (!row_ok || nt <= 0) continue;
        if (p.n_splits > 1) {
          float* dst = p.partial + (((int64_t)w.split * p.batch + w.bz) * p.N + w.n0 + c) * p.M + m;
#pragma unroll
          for (int jj = 0; jj < 32; ++jj)
            if (jj < nt) dst[(int64_t)jj * p.M] = w.nk > 0 ? __uint_as_float(r[jj]) : 0.f;
          continue;
        }
        const int64_t o0 = w.bz * p.out_sb + (int64_t)(w.n0 + c) * p.out_st + m;
        const int64_t g0 = w.bz * p.gate_sb + (int64_t)(w.n0 + c) * p.gate_st + m;
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          if (jj >= nt) break;
          float v = w.nk > 0 ? __uint_as_float(r[jj]) : 0.f;
          if (p.sigmoid) v = 1.f / (1.f + expf(-v));
          if (p.gate) v *= __bfloat162float(p.gate[g0 + (int64_t)jj * p.gate_st]);
          if (p.out_f32)
            static_cast<float*>(p.out)[o0 + (int64_t)jj * p.out_st] = v;
          else
            static_cast<__nv_bfloat16*>(p.out)[o0 + (int64_t)jj * p.out_st] = __float2bfloat16_rn(v);
        }
      }
      if (p.tail && w.m0 == 0 && w.split == 0) {
        // the tail columns of this unit's tokens (16-byte chunks; the host checks the alignment)
        const int cpr = p.tail_cols / 8;
        for (int idx = et; idx < BN * cpr; idx += 128) {
          const int t = w.n0 + idx / cpr, q = idx % cpr;
          if (t >= p.N) break;
          const uint4 v = reinterpret_cast<const uint4*>(p.tail + w.bz * p.tail_sb + (int64_t)t * p.tail_st)[q];
          reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + w.bz * p.out_sb + (int64_t)t * p.out_st +
                                   p.tail_off)[q] = v;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);       // this warp's rows of the accumulator are read
    }
  }

  // ---- teardown: nothing of this CTA's may be in flight when its tensor memory is released ----
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t drain_ns = p.wait_ns > 100000000ull ? p.wait_ns : 100000000ull;
    if (*abort_flag) {
      // only the last load of a stage can still be in flight (a later one waited for the MMAs to read
      // the earlier)
      for (int s = 0; s < STAGES; ++s) {
        const int g = last_load[s];
        if (g >= 0) (void)mbar_wait(&full[s], (uint32_t)((g / STAGES) & 1), drain_ns, p.status);
      }
    }
    (void)mbar_wait(done, 0, drain_ns, p.status);      // the MMA issuer's final commit
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, PCfg::TMEM_COLS);
  }
}

struct GemmOperand {
  // a 3-D bf16 tensor seen as [batch][rows][k] (K-major) or [batch][k][rows] (MN-major)
  void* base;
  uint64_t inner, mid, outer;            // dims from innermost
  uint64_t stride_mid, stride_outer;     // bytes
};

struct GemmPlan {
  int BN, n_tiles, m_tiles, splits, k_chunks;
  bool persistent;   // the persistent kernel (several units per CTA) instead of one tile per CTA
};

// Tiling of out[bz][t][m] = sum_k A[bz](m, k) B[bz](t, k): 128-row tiles of A, BN-token tiles of B,
// and K split into `splits` ranges. Products with more tiles than SMs and at least 8 K chunks per tile
// (the dense linears of a prefill) run on the persistent kernel, the K splits chosen by a cost in K
// chunks on the busiest SM (a split adds the sum kernel, about 7 chunks' time, and the partials'
// traffic). The others keep one tile (and K range) per CTA, split along K until one wave of tiles
// covers the SMs: their CTAs are short, and several run at once on an SM.
static GemmPlan plan_gemm(int M, int N, int K, int batch, int max_splits) {
  GemmPlan g;
  g.BN = N <= 64 ? 64 : (N <= 128 ? 128 : 256);
  g.n_tiles = (int)ceil_div(N, g.BN);
  g.m_tiles = (int)ceil_div(M, 128);
  const int total_chunks = (int)ceil_div(K, 64);
  const int64_t base = (int64_t)g.m_tiles * g.n_tiles * batch;
  const int64_t G = sm_count();
  g.persistent = base > G && total_chunks >= 8;
  int best = 1;
  if (g.persistent) {
    const double stage_bytes = 128.0 * 64 * 2 + g.BN * 64.0 * 2;
    double best_cost = (double)ceil_div(base, G) * total_chunks;
    const int s_max = std::min(std::max(1, max_splits), std::min(total_chunks / 2, 32));
    for (int s = 2; s <= s_max; ++s) {
      const int kc = (int)ceil_div(total_chunks, s);
      const int ss = (int)ceil_div(total_chunks, kc);
      const double cost = (double)ceil_div(base * ss, G) * kc + 7.0 +
                          2.0 * ss * batch * (double)N * M * 4.0 / ((double)G * stage_bytes);
      if (cost < best_cost) {
        best_cost = cost;
        best = ss;
      }
    }
  } else {
    best = (int)std::max<int64_t>(1, std::min<int64_t>(G / std::max<int64_t>(base, 1), total_chunks / 4));
    best = std::min(best, std::max(1, max_splits));
  }
  g.k_chunks = (int)ceil_div(total_chunks, best);
  g.splits = (int)ceil_div(total_chunks, g.k_chunks);
  return g;
}

static size_t gemm_partial_bytes(int M, int N, int K, int batch) {
  GemmPlan g = plan_gemm(M, N, K, batch, 1 << 20);
  return g.splits > 1 ? round_up((size_t)g.splits * batch * N * M * sizeof(float), 256) : 0;
}

template <int BN, bool A_MN>
static int launch_gemm_wave_t(const CUtensorMap& ta, const CUtensorMap& tb, TcGemmParams p, cudaStream_t s) {
  static bool attr_set[64] = {false};
  const int dev = current_device();
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(tc_gemm_kernel<BN, A_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmCfg<BN>::SMEM) != cudaSuccess)
      return MLA_ERR_CUDA;
    attr_set[dev] = true;
  }
  const dim3 grid((unsigned)p.m_tiles, (unsigned)(p.n_tiles * p.n_splits), (unsigned)p.batch);
  if (grid.y > 65535u || grid.z > 65535u) return MLA_ERR_UNSUPPORTED;
  // a ring no deeper than the K chunks of one CTA: short-K products then fit several CTAs per SM
  p.stages = std::max(1, std::min(GemmCfg<BN>::STAGES, p.k_chunks));
  const int smem = p.stages * GemmCfg<BN>::STAGE + 1024 + 256;
  return launch_pdl(tc_gemm_kernel<BN, A_MN>, grid, dim3(128), (size_t)smem, s, ta, tb, p);
}

template <int BN, bool A_MN>
static int launch_gemm_t(const CUtensorMap& ta, const CUtensorMap& tb, TcGemmParams p, cudaStream_t s,
                         bool persistent) {
  if (!persistent) return launch_gemm_wave_t<BN, A_MN>(ta, tb, p, s);
  using PCfg = GemmPCfg<BN>;
  static bool attr_set[64] = {false};
  const int dev = current_device();
  const int smem_max = PCfg::STAGES * GemmCfg<BN>::STAGE + PCfg::FIXED;
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(tc_gemm_persistent_kernel<BN, A_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_max) != cudaSuccess)
      return MLA_ERR_CUDA;
    attr_set[dev] = true;
  }
  const int64_t U = (int64_t)p.m_tiles * p.n_tiles * p.n_splits * p.batch;
  const int64_t G = std::min<int64_t>(U, sm_count());
  // a ring no deeper than the chunks one CTA streams
  const int64_t chunks_per_cta = ceil_div(U, G) * p.k_chunks;
  p.stages = (int)std::max<int64_t>(2, std::min<int64_t>(PCfg::STAGES, chunks_per_cta));
  const int smem = p.stages * GemmCfg<BN>::STAGE + PCfg::FIXED;
  return launch_pdl(tc_gemm_persistent_kernel<BN, A_MN>, dim3((unsigned)G), dim3(GEMM_P_THREADS), (size_t)smem, s,
                    ta, tb, p);
}

// out[bz][t][m] = epi(sum_k A[bz](m, k) B[bz](t, k)); A MN-major when a_mn
struct GemmTail {
  const void* src = nullptr;
  int64_t sb = 0, st = 0, off = 0;
  int cols = 0;
};

// sum_partials = false: a K-split product leaves its fp32 partials [split][batch][N][M] in partial_ws for
// the consumer to add in split order (the consumer then reads partial_ws with gemm_splits() parts)
static int tc_gemm(const GemmOperand& A, bool a_mn, const GemmOperand& Bop, int M, int N, int K, int batch,
                   void* out, int64_t out_sb, int64_t out_st, bool out_f32, const void* gate, int64_t gate_sb,
                   int64_t gate_st, bool sigmoid, void* partial_ws, cudaStream_t s,
                   const GemmTail& tail = GemmTail(), bool sum_partials = true) {
  // a K-major A may end inside its last 128-row tile (the TMA zero-fills the rows past M and the
  // epilogue skips them); an MN-major A loads its rows as 64-wide boxes and takes whole tiles only
  if (M <= 0 || M % 4 || (a_mn && M % 128) || K % 64 || N <= 0 || batch <= 0) return MLA_ERR_UNSUPPORTED;
  // the epilogue writes runs of 4 consecutive outputs (8 or 16 bytes) and reads 4 gate values
  if (out_sb % 4 || out_st % 4 || (reinterpret_cast<uintptr_t>(out) & 15) ||
      (gate && (gate_sb % 4 || gate_st % 4 || (reinterpret_cast<uintptr_t>(gate) & 7))))
    return MLA_ERR_UNSUPPORTED;
  const GemmPlan g = plan_gemm(M, N, K, batch, partial_ws ? (1 << 20) : 1);
  CUtensorMap ta, tb;
  {
    const uint64_t dims[3] = {A.inner, A.mid, A.outer};
    const uint64_t st[2] = {A.stride_mid, A.stride_outer};
    const uint32_t box[3] = {64, a_mn ? 64u : 128u, 1};
    if (!encode_tmap_bf16(&ta, A.base, 3, dims, st, box)) return MLA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {Bop.inner, Bop.mid, Bop.outer};
    const uint64_t st[2] = {Bop.stride_mid, Bop.stride_outer};
    const uint32_t box[3] = {64, (uint32_t)g.BN, 1};
    if (!encode_tmap_bf16(&tb, Bop.base, 3, dims, st, box)) return MLA_ERR_CUDA;
  }
  TcGemmParams p{};
  p.M = M; p.N = N; p.K = K; p.m_tiles = g.m_tiles; p.n_tiles = g.n_tiles; p.k_chunks = g.k_chunks;
  p.n_splits = g.splits;
  p.batch = batch; p.out = out; p.out_sb = out_sb; p.out_st = out_st; p.out_f32 = out_f32 ? 1 : 0;
  p.gate = static_cast<const __nv_bfloat16*>(gate); p.gate_sb = gate_sb; p.gate_st = gate_st;
  p.partial = static_cast<float*>(partial_ws); p.sigmoid = sigmoid ? 1 : 0;
  if (tail.src && tail.cols > 0) {
    if (out_f32 || tail.cols % 8 || tail.sb % 8 || tail.st % 8 || tail.off % 8 || out_sb % 8 || out_st % 8 ||
        (reinterpret_cast<uintptr_t>(tail.src) & 15) || (reinterpret_cast<uintptr_t>(out) & 15))
      return MLA_ERR_UNSUPPORTED;
    p.tail = static_cast<const __nv_bfloat16*>(tail.src);
    p.tail_sb = tail.sb; p.tail_st = tail.st; p.tail_off = tail.off; p.tail_cols = tail.cols;
  }
  p.status = device_status_ptr(); p.wait_ns = (unsigned long long)wait_limit();
  if (!p.status) return MLA_ERR_CUDA;
  if (g.splits > 1 && !partial_ws) return MLA_ERR_WORKSPACE;
  if ((int64_t)g.m_tiles * g.n_tiles * g.splits * batch >= (1LL << 31)) return MLA_ERR_UNSUPPORTED;
  int st;
  const bool pk = g.persistent;
  if (a_mn) {
    st = g.BN == 64 ? launch_gemm_t<64, true>(ta, tb, p, s, pk)
                    : g.BN == 128 ? launch_gemm_t<128, true>(ta, tb, p, s, pk)
                                  : launch_gemm_t<256, true>(ta, tb, p, s, pk);
  } else {
    st = g.BN == 64 ? launch_gemm_t<64, false>(ta, tb, p, s, pk)
                    : g.BN == 128 ? launch_gemm_t<128, false>(ta, tb, p, s, pk)
                                  : launch_gemm_t<256, false>(ta, tb, p, s, pk);
  }
  if (st) return st;
  if (g.splits > 1 && sum_partials) {
    const int64_t per = (int64_t)batch * N * M;
    const unsigned blocks = (unsigned)std::min<int64_t>(ceil_div(per / 4, 128), 16 * sm_count());
    st = launch_pdl(splitk_reduce_kernel, dim3(blocks), dim3(128), 0, s, (const float*)p.partial, g.splits, batch,
                    N, M, out, (int64_t)out_sb, (int64_t)out_st, p.out_f32, p.gate, (int64_t)gate_sb,
                    (int64_t)gate_st, p.sigmoid);
    if (st) return st;
  }
  return MLA_OK;
}

// ---------------------------------------------------------------------------------------------
// the library's products on the tensor-core GEMM
// ---------------------------------------------------------------------------------------------
bool tc_absorb_supported(const mla_dims& d, int64_t n_rows) {
  return d.kv_lora_rank % 128 == 0 && d.qk_nope % 64 == 0 && d.qk_nope > 0 && n_rows > 0 &&
         n_rows < (1LL << 30) && ((int64_t)d.n_heads * d.qk_nope * 2) % 16 == 0 &&
         ((int64_t)d.kv_lora_rank * 2) % 16 == 0 && d.rope_dim % 8 == 0;
}

int tc_absorb_query(const mla_dims& d, const void* q_nope, const void* q_pe, const void* w_uk, int64_t n_rows,
                    void* q_abs, cudaStream_t s) {
  const int64_t H = d.n_heads, n = d.qk_nope, dc = d.kv_lora_rank, dr = d.rope_dim, W = dc + dr;
  // A = W_UK[h] viewed as (m = j, k = i): MN-major, tensor [H][n][dc]
  GemmOperand A{const_cast<void*>(w_uk), (uint64_t)dc, (uint64_t)n, (uint64_t)H, (uint64_t)(dc * 2),
                (uint64_t)(n * dc * 2)};
  // B = q_nope[:, h, :]: tensor [rows][H][n] seen as (k = i, t, h)
  GemmOperand B{const_cast<void*>(q_nope), (uint64_t)n, (uint64_t)n_rows, (uint64_t)H, (uint64_t)(H * n * 2),
                (uint64_t)(n * 2)};
  // the rotary tail q_abs[t, h, d_c:] = q_pe[t, h] is copied by the same kernel
  GemmTail tail;
  if (dr > 0) {
    tail.src = q_pe; tail.sb = dr; tail.st = H * dr; tail.off = dc; tail.cols = (int)dr;
  }
  return tc_gemm(A, true, B, (int)dc, (int)n_rows, (int)n, (int)H, q_abs, W, H * W, false, nullptr, 0, 0,
                 false, nullptr, s, tail);
}

bool tc_out_project_supported(const mla_dims& d, int64_t n_rows) {
  const int64_t H = d.n_heads, dc = d.kv_lora_rank, dv = d.v_head, D = d.d_model;
  return dv % 128 == 0 && dc % 64 == 0 && D % 128 == 0 && (H * dv) % 64 == 0 && n_rows > 0 &&
         n_rows < (1LL << 30) && dc % 4 == 0;
}

// scratch beyond v: out_lat in bf16, then the split-K partials of the output projection
size_t tc_out_project_extra_workspace(const mla_dims& d, int64_t n_rows) {
  if (!tc_out_project_supported(d, n_rows)) return 0;
  const int64_t H = d.n_heads, dc = d.kv_lora_rank, dv = d.v_head, D = d.d_model;
  return round_up((size_t)n_rows * H * dc * 2, 256) + gemm_partial_bytes((int)D, (int)n_rows, (int)(H * dv), 1);
}

int tc_out_project(const mla_dims& d, const void* out_lat, bool lat_bf16, const void* w_uv, const void* w_o,
                   const void* gate, int64_t n_rows, void* y, void* workspace, size_t ws_bytes, cudaStream_t s) {
  const int64_t H = d.n_heads, dc = d.kv_lora_rank, dv = d.v_head, D = d.d_model;
  char* ws = static_cast<char*>(workspace);
  void* v = ws;
  const size_t v_bytes = round_up((size_t)n_rows * H * dv * 2, 256);
  void* lat16 = lat_bf16 ? const_cast<void*>(out_lat) : static_cast<void*>(ws + v_bytes);
  const size_t lat_bytes = round_up((size_t)n_rows * H * dc * 2, 256);
  void* partial = ws + v_bytes + lat_bytes;
  if (ws_bytes < v_bytes + tc_out_project_extra_workspace(d, n_rows)) return MLA_ERR_WORKSPACE;
  if (!lat_bf16) {
    // the W_UV GEMM reads out_lat as its bf16 B operand
    const int64_t n4 = n_rows * H * dc / 4;
    const unsigned blocks = (unsigned)std::min<int64_t>(ceil_div(n4, 256), 8 * sm_count());
    const int st0 = launch_pdl(f32_to_bf16_kernel, dim3(blocks), dim3(256), 0, s,
                               static_cast<const float4*>(out_lat), static_cast<uint2*>(lat16), n4);
    if (st0) return st0;
  }
  // v[t, h, i] = gate * sum_j W_UV[h, i, j] lat[t, h, j]: A = W_UV[h] K-major, B = lat[:, h, :]
  GemmOperand A1{const_cast<void*>(w_uv), (uint64_t)dc, (uint64_t)dv, (uint64_t)H, (uint64_t)(dc * 2),
                 (uint64_t)(dv * dc * 2)};
  GemmOperand B1{lat16, (uint64_t)dc, (uint64_t)n_rows, (uint64_t)H, (uint64_t)(H * dc * 2), (uint64_t)(dc * 2)};
  int st = tc_gemm(A1, false, B1, (int)dv, (int)n_rows, (int)dc, (int)H, v, dv, H * dv, false, gate, dv, H * dv,
                   false, nullptr, s);
  if (st) return st;
  // y[t, o] = sum_k W_O[o, k] v[t, k]
  const int64_t K = H * dv;
  GemmOperand A2{const_cast<void*>(w_o), (uint64_t)K, (uint64_t)D, 1, (uint64_t)(K * 2), (uint64_t)(D * K * 2)};
  GemmOperand B2{v, (uint64_t)K, (uint64_t)n_rows, 1, (uint64_t)(K * 2), (uint64_t)(n_rows * K * 2)};
  return tc_gemm(A2, false, B2, (int)D, (int)n_rows, (int)K, 1, y, 0, D, false, nullptr, 0, 0, false, partial, s);
}

// ---------------------------------------------------------------------------------------------
// input projections: c' = x W_cq^T (bf16 scratch), q_nope = c' W_qc^T (bf16), q_r = c' W_qr^T (fp32),
// kv = x W_dkv^T (fp32). A = the weight (K-major, M = its output rows), B = the activations.
// ---------------------------------------------------------------------------------------------
bool tc_project_supported(const mla_dims& d, int64_t q_rank, int64_t n_rows) {
  const int64_t H = d.n_heads, n = d.qk_nope, dr = d.rope_dim, dc = d.kv_lora_rank, D = d.d_model;
  return n_rows > 0 && n_rows < (1LL << 30) && D % 64 == 0 && q_rank % 64 == 0 && q_rank < (1LL << 30) &&
         n > 0 && (H * n) % 4 == 0 && (H * dr) % 4 == 0 && (dc + dr) % 4 == 0 && H * n < (1LL << 30) &&
         D < (1LL << 30);
}

static void project_gemm_dims(const mla_dims& d, int64_t q_rank, int64_t n_rows, int dims[4][3]) {
  const int64_t H = d.n_heads;
  const int64_t rows[4] = {q_rank, H * d.qk_nope, H * d.rope_dim, (int64_t)d.kv_lora_rank + d.rope_dim};
  const int64_t ks[4] = {d.d_model, q_rank, q_rank, d.d_model};
  for (int i = 0; i < 4; ++i) {
    dims[i][0] = (int)rows[i]; dims[i][1] = (int)n_rows; dims[i][2] = (int)ks[i];
  }
}

// split-K scratch of the four products, one region each: the rotary-query partials are read
// later, by the rotation kernel
static void project_partial_offsets(const mla_dims& d, int64_t q_rank, int64_t n_rows, size_t off[5]) {
  int g[4][3];
  project_gemm_dims(d, q_rank, n_rows, g);
  off[0] = 0;
  for (int i = 0; i < 4; ++i) off[i + 1] = off[i] + (g[i][0] > 0 ? gemm_partial_bytes(g[i][0], g[i][1], g[i][2], 1) : 0);
}

size_t tc_project_partial_bytes(const mla_dims& d, int64_t q_rank, int64_t n_rows) {
  size_t off[5];
  project_partial_offsets(d, q_rank, n_rows, off);
  return off[4];
}

int tc_project(const mla_dims& d, int64_t q_rank, const void* x, const void* w_cq, const void* w_qc,
               const void* w_qr, const void* w_dkv, int64_t n_rows, void* c_q, void* q_nope, float* q_r,
               float* kv, void* partial, cudaStream_t s, ProjectParts* parts, cudaStream_t s_kv) {
  int g[4][3];
  project_gemm_dims(d, q_rank, n_rows, g);
  size_t off[5];
  project_partial_offsets(d, q_rank, n_rows, off);
  char* pw = static_cast<char*>(partial);
  // the rotary-query product leaves its K-split partials to the rotation, which adds them in order
  // (the KV product keeps its own reduce: the append runs one block per token and would read the
  // partials with too few threads)
  const int qr_splits = g[2][0] > 0 ? plan_gemm(g[2][0], g[2][1], g[2][2], 1, 1 << 20).splits : 1;
  parts->qr = qr_splits > 1 ? reinterpret_cast<const float*>(pw + off[2]) : q_r;
  parts->qr_parts = qr_splits;
  parts->qr_stride = (int64_t)g[2][1] * g[2][0];
  const int64_t D = d.d_model;
  auto weight = [](const void* w, int64_t rows, int64_t k) {
    return GemmOperand{const_cast<void*>(w), (uint64_t)k, (uint64_t)rows, 1, (uint64_t)(k * 2),
                       (uint64_t)(rows * k * 2)};
  };
  const GemmOperand bx{const_cast<void*>(x), (uint64_t)D, (uint64_t)n_rows, 1, (uint64_t)(D * 2),
                       (uint64_t)(n_rows * D * 2)};
  const GemmOperand bq{c_q, (uint64_t)q_rank, (uint64_t)n_rows, 1, (uint64_t)(q_rank * 2),
                       (uint64_t)(n_rows * q_rank * 2)};
  // the KV down-projection (on s_kv), then the query chain (c_q feeds the last two products)
  int st = tc_gemm(weight(w_dkv, g[3][0], D), false, bx, g[3][0], g[3][1], g[3][2], 1, kv, 0, g[3][0], true,
                   nullptr, 0, 0, false, pw + off[3], s_kv);
  if (st) return st;
  if ((st = tc_gemm(weight(w_cq, g[0][0], D), false, bx, g[0][0], g[0][1], g[0][2], 1, c_q, 0, g[0][0], false,
                    nullptr, 0, 0, false, pw + off[0], s)))
    return st;
  if ((st = tc_gemm(weight(w_qc, g[1][0], q_rank), false, bq, g[1][0], g[1][1], g[1][2], 1, q_nope, 0, g[1][0],
                    false, nullptr, 0, 0, false, pw + off[1], s)))
    return st;
  if (g[2][0] > 0)
    st = tc_gemm(weight(w_qr, g[2][0], q_rank), false, bq, g[2][0], g[2][1], g[2][2], 1, q_r, 0, g[2][0], true,
                 nullptr, 0, 0, false, pw + off[2], s, GemmTail(), false);
  return st;
}

bool tc_linear_supported(int64_t m, int64_t n, int64_t k) {
  return n % 128 == 0 && k % 64 == 0 && m > 0 && m < (1LL << 30) && n < (1LL << 30) && k < (1LL << 30) &&
         gemm_partial_bytes((int)n, (int)m, (int)k, 1) == 0;
}

int tc_linear(const void* x, const void* w, int64_t m, int64_t n, int64_t k, int sigmoid, void* y, cudaStream_t s) {
  // Y[t, o] = sum_k W[o, k] X[t, k]: A = W (M = n), B = X (N = m)
  GemmOperand A{const_cast<void*>(w), (uint64_t)k, (uint64_t)n, 1, (uint64_t)(k * 2), (uint64_t)(n * k * 2)};
  GemmOperand B{const_cast<void*>(x), (uint64_t)k, (uint64_t)m, 1, (uint64_t)(k * 2), (uint64_t)(m * k * 2)};
  return tc_gemm(A, false, B, (int)n, (int)m, (int)k, 1, y, 0, n, false, nullptr, 0, 0, sigmoid != 0, nullptr, s);
}

}  // namespace mla
