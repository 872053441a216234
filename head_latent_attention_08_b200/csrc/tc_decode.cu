// tc_decode.cu -- fused split-KV absorbed-MLA decode on sm_100a tensor cores.
//
// What it computes ("ferrox-core 0.23.0 src/mla_absorbed.rs", module docs "What it is"):
//   score[r][t] = (q_abs[r] . c[t] + q_pe[r] . k_pe[t]) * kq_scale,
//   out_lat[r]  = sum_t softmax_t(score[r]) c[t]           (kv_lora_rank = 512 wide)
// for every query row r = (query token j, head h) of a sequence, over the positions t it sees
// (all of them, or t <= T - n_q + j under the causal mask of "Gated MLA", Hint 2).
//
// Design (B200):
//  * Rows: 128 consecutive rows of q_abs form one M = 128 block (all 128 heads of one query token at
//    DeepSeek-V2 scale; 8 tokens x 16 heads in gated prefill). Every row of a block shares the key row
//    [c_t | k_pe_t] and the value c_t, so QK^T and P.C are dense 128-row MMAs.
//  * TMEM cannot hold O (128 x 512 fp32 = all 512 columns) next to S, so a CLUSTER OF TWO CTAs shares
//    one block: CTA 0 owns latent dims [0, 256), CTA 1 owns [256, 512) plus the 64 rotary dims. Each
//    streams only its own columns of every cache tile (each cache byte crosses HBM once), computes the
//    partial S over its columns on tcgen05 into TMEM, and the two partials are exchanged through
//    distributed shared memory and summed (both CTAs form bit-identical S = S0 + S1). Each CTA then
//    runs the same fp32 online softmax and accumulates its half of O = P . C in TMEM (256 columns).
//  * P (bf16) is written back into the TMEM columns of its own S tile and used as the A operand of
//    the P . C MMA straight from TMEM. S is double-buffered, so QK^T of tile i+1 overlaps the softmax
//    of tile i.
//  * O is rescaled only when a row's running maximum grows by more than 2^8 (the result is exact:
//    numerator and denominator share the stale reference maximum).
//  * Work: the (block, 64-position tile) units of all sequences are split evenly over the clusters
//    (persistent, one cluster per SM pair). A cluster that covers a whole block writes the normalised
//    result; split blocks leave (O, max, sum) partials that a combine kernel merges.
//  * Warp roles per CTA (256 threads): warp 0 lane 0 issues TMA loads, warp 1 lane 0 issues MMAs,
//    warps 4-7 (one thread per row / TMEM lane) run the softmax, the exchange and the epilogue.
//  * Every wait is bounded (global-timer limit); a wait that gives up sets the library's status word,
//    and the CTA abandons its work, drains its own TMA loads and exits through the cluster barrier.
#include <math.h>

#include <algorithm>

#include "sm100.cuh"
#include "tc.cuh"

namespace mla {

using namespace sm100;

constexpr int DEC_BT = 64;          // positions per tile
constexpr int DEC_THREADS = 256;
constexpr int DEC_DC = 512;         // latent width handled by this kernel
constexpr int DEC_HALF = 256;       // latent columns per CTA
constexpr int DEC_ROWS = 128;       // rows per block

template <int DR>
struct DecCfg {
  static constexpr int KA_MAX = 4 + DR / 64;            // 64-wide column boxes of CTA 1
  static constexpr int Q_BOX = 128 * 128;               // 128 rows x 128 B
  static constexpr int K_BOX = DEC_BT * 128;            // 64 rows x 128 B
  static constexpr int Q_BYTES = KA_MAX * Q_BOX;
  static constexpr int STAGE_BYTES = KA_MAX * K_BOX;
  static constexpr int STAGES = DR == 0 ? 3 : 2;
  static constexpr int X_SLOT = DEC_ROWS * DEC_BT * 4;  // one partial S tile, fp32
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_X = OFF_K + STAGES * STAGE_BYTES;
  static constexpr int OFF_BAR = OFF_X + 2 * X_SLOT;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
};

struct DecParams {
  const int32_t* cu;
  int32_t batch, n_q, H, nbps, nblocks;
  int64_t total_rows;
  int causal;
  float scale_log2;           // kq_scale * log2(e)
  const int32_t* prefix;      // [nblocks + 1] exclusive prefix of tiles per block
  int G;                      // clusters
  float* out_lat;
  float* lse;
  float* o_part;              // [2G][128][512]
  float* m_part;              // [2G][128] reference maxima (log2 domain)
  float* l_part;              // [2G][128] sums
  int* status;
  unsigned long long wait_ns;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// sequence bounds clamped to the cache
__device__ __forceinline__ void seq_bounds(const DecParams& p, int b, int64_t& start, int& T) {
  const int64_t c0 = p.cu[b], c1 = p.cu[b + 1];
  const int64_t s = c0 < 0 ? 0 : (c0 > p.total_rows ? p.total_rows : c0);
  const int64_t e = c1 < s ? s : (c1 > p.total_rows ? p.total_rows : c1);
  start = s;
  T = (int)(e - s);
}

// tiles a block needs: up to the last position its last valid row sees
__device__ __forceinline__ int block_tiles(int T, int n_q, int H, int rb, int causal) {
  const int rows = n_q * H;
  const int last_row = min(rows - 1, rb * DEC_ROWS + DEC_ROWS - 1);
  int cnt = T;
  if (causal) {
    const int j = last_row / H;
    cnt = T - n_q + j + 1;
    cnt = cnt < 0 ? 0 : (cnt > T ? T : cnt);
  }
  return (cnt + DEC_BT - 1) / DEC_BT;
}

// largest k with prefix[k] <= u (the non-empty block that holds unit u, u < prefix[n])
__device__ __forceinline__ int find_block(const int32_t* prefix, int n, int64_t u) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int64_t)prefix[mid] <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int64_t range_start(int64_t U, int G, int p) { return (int64_t)p * U / G; }

// largest p with range_start(p) <= u
__device__ __forceinline__ int find_owner(int64_t U, int G, int64_t u) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (range_start(U, G, mid) <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ---------------------------------------------------------------------------------------------
// plan: tiles per block and their exclusive prefix (one CTA)
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) decode_plan_kernel(DecParams p, int32_t* prefix) {
  __shared__ int64_t sums[1024];
  const int n = p.nblocks;
  const int per = (n + 1023) / 1024;
  const int k0 = threadIdx.x * per, k1 = min(n, k0 + per);
  int64_t local = 0;
  for (int k = k0; k < k1; ++k) {
    int64_t s; int T;
    seq_bounds(p, k / p.nbps, s, T);
    local += block_tiles(T, p.n_q, p.H, k % p.nbps, p.causal);
  }
  sums[threadIdx.x] = local;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const int64_t v = threadIdx.x >= off ? sums[threadIdx.x - off] : 0;
    __syncthreads();
    sums[threadIdx.x] += v;
    __syncthreads();
  }
  int64_t run = sums[threadIdx.x] - local;   // exclusive
  for (int k = k0; k < k1; ++k) {
    prefix[k] = (int32_t)run;
    int64_t s; int T;
    seq_bounds(p, k / p.nbps, s, T);
    run += block_tiles(T, p.n_q, p.H, k % p.nbps, p.causal);
  }
  if (threadIdx.x == 1023) prefix[n] = (int32_t)sums[1023];
}

// ---------------------------------------------------------------------------------------------
// the decode kernel
// ---------------------------------------------------------------------------------------------
template <int DR>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(DEC_THREADS, 1)
    tc_decode_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     DecParams p) {
  using Cfg = DecCfg<DR>;
  constexpr int ST = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + Cfg::OFF_Q;
  uint8_t* sK = smem + Cfg::OFF_K;
  float* sX = reinterpret_cast<float*>(smem + Cfg::OFF_X);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* k_full = bars;
  uint64_t* k_empty = k_full + ST;
  uint64_t* q_full = k_empty + ST;
  uint64_t* q_empty = q_full + 1;
  uint64_t* s_full = q_empty + 1;     // [2]
  uint64_t* p_full = s_full + 2;      // [2]
  uint64_t* o_done = p_full + 2;      // [1]
  uint64_t* x_full = o_done + 1;      // [2]
  uint64_t* x_empty = x_full + 2;     // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(x_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int pair = blockIdx.x >> 1;
  const int KA = rank == 0 ? 4 : 4 + DR / 64;
  const int dim0 = rank == 0 ? 0 : DEC_HALF;

  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&x_full[s], 128);
      mbar_init(&x_empty[s], 128);
    }
    mbar_init(o_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tq);
    prefetch_tmap(&tk);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();           // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tO = tmem;               // columns [0, 256): this CTA's half of O
  const uint32_t tS = tmem + 256;         // columns [256, 384): two 64-column S / P tiles

  const int64_t U = p.prefix[p.nblocks];
  const int64_t u0 = range_start(U, p.G, pair), u1 = range_start(U, p.G, pair + 1);
  const int64_t drain_ns = p.wait_ns > 100000000ull ? p.wait_ns : 100000000ull;

  if (warp == 0 && lane == 0) {
    // ------------------------------- TMA producer -------------------------------
    int64_t g = 0;
    int seg = 0;
    int q_loads = 0;
    int64_t u = u0;
    int k = u0 < u1 ? find_block(p.prefix, p.nblocks, u0) : 0;
    bool ok = true;
    while (u < u1 && ok) {
      const int64_t bstart = p.prefix[k], bend = p.prefix[k + 1];
      const int64_t send = u1 < bend ? u1 : bend;
      const int tile0 = (int)(u - bstart), ntl = (int)(send - u);
      const int b = k / p.nbps, rb = k % p.nbps;
      int64_t sstart; int T;
      seq_bounds(p, b, sstart, T);
      const int qrow = (int)((int64_t)b * p.n_q * p.H + (int64_t)rb * DEC_ROWS);
      if (seg > 0 && (*abort_flag || !mbar_wait(q_empty, (seg - 1) & 1, p.wait_ns, p.status))) { ok = false; break; }
      mbar_arrive_expect_tx(q_full, KA * Cfg::Q_BOX);
      for (int kb = 0; kb < KA; ++kb) tma_load_2d(sQ + kb * Cfg::Q_BOX, &tq, q_full, dim0 + kb * 64, qrow);
      ++q_loads;
      for (int tt = 0; tt < ntl; ++tt, ++g) {
        const int s = (int)(g % ST);
        if (g >= ST && (*abort_flag || !mbar_wait(&k_empty[s], (int)((g / ST) - 1) & 1, p.wait_ns, p.status))) {
          ok = false;
          break;
        }
        uint8_t* dst = sK + s * Cfg::STAGE_BYTES;
        mbar_arrive_expect_tx(&k_full[s], KA * Cfg::K_BOX);
        const int y = (int)(sstart + (int64_t)(tile0 + tt) * DEC_BT);
        for (int kb = 0; kb < KA; ++kb) tma_load_2d(dst + kb * Cfg::K_BOX, &tk, &k_full[s], dim0 + kb * 64, y);
      }
      u = send;
      ++seg;
      if (u < u1) k = find_block(p.prefix, p.nblocks, u);
    }
    if (!ok) *abort_flag = 1;
    if (*abort_flag) {
      // drain this CTA's own loads in flight before the shared memory is released
      for (int64_t i = (g > ST ? g - ST : 0); i < g; ++i)
        (void)mbar_wait(&k_full[i % ST], (int)(i / ST) & 1, drain_ns, p.status);
      if (q_loads > 0) (void)mbar_wait(q_full, (q_loads - 1) & 1, drain_ns, p.status);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------- MMA issuer -------------------------------
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, DEC_BT, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, DEC_HALF, false, true);
    const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK);
    int64_t g = 0;
    int seg = 0;
    bool have_prev = false, prev_first = false;
    int64_t prev_g = 0;
    bool ok = true;
    auto issue_pv = [&](int64_t pg, bool first) -> bool {
      const int sl = (int)(pg & 1);
      if (*abort_flag || !mbar_wait(&p_full[sl], (int)(pg >> 1) & 1, p.wait_ns, p.status)) return false;
      tc_fence_after();
      const int s = (int)(pg % ST);
      const uint32_t c_base = k_base + s * Cfg::STAGE_BYTES;
#pragma unroll
      for (int kk = 0; kk < DEC_BT / 16; ++kk) {
        const uint64_t bd = smem_desc_sw128(c_base + kk * 2048, Cfg::K_BOX, 1024);
        mma_bf16_ts(tO, tS + sl * 64 + kk * 8, bd, idesc_pv, (first && kk == 0) ? 0u : 1u);
      }
      mma_commit(&k_empty[s]);
      mma_commit(o_done);
      return true;
    };
    int64_t u = u0;
    int k = u0 < u1 ? find_block(p.prefix, p.nblocks, u0) : 0;
    while (u < u1 && ok) {
      const int64_t bend = p.prefix[k + 1];
      const int64_t send = u1 < bend ? u1 : bend;
      const int ntl = (int)(send - u);
      if (*abort_flag || !mbar_wait(q_full, seg & 1, p.wait_ns, p.status)) { ok = false; break; }
      tc_fence_after();
      for (int tt = 0; tt < ntl; ++tt, ++g) {
        const int s = (int)(g % ST);
        const int sl = (int)(g & 1);
        if (*abort_flag || !mbar_wait(&k_full[s], (int)(g / ST) & 1, p.wait_ns, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kst = k_base + s * Cfg::STAGE_BYTES;
        for (int kb = 0; kb < KA; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc_sw128(q_base + kb * Cfg::Q_BOX + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(kst + kb * Cfg::K_BOX + kk * 32, 16, 1024);
            mma_bf16_ss(tS + sl * 64, ad, bd, idesc_qk, (kb | kk) ? 1u : 0u);
          }
        }
        mma_commit(&s_full[sl]);
        if (tt == ntl - 1) mma_commit(q_empty);
        if (have_prev && !issue_pv(prev_g, prev_first)) { ok = false; break; }
        have_prev = true;
        prev_g = g;
        prev_first = (tt == 0);
      }
      u = send;
      ++seg;
      if (u < u1) k = find_block(p.prefix, p.nblocks, u);
    }
    if (ok && have_prev) ok = issue_pv(prev_g, prev_first);
    if (!ok) *abort_flag = 1;
  } else if (warp >= 4) {
    // ---------------------- softmax, exchange and epilogue ----------------------
    const int row = tid - 128;                         // TMEM lane = block row
    const uint32_t lane_off = (uint32_t)((warp - 4) * 32) << 16;
    const uint32_t x_local = smem_u32(sX);
    const uint32_t x_remote = map_to_cta(x_local, peer);
    const uint32_t xf_remote = map_to_cta(smem_u32(x_full), peer);
    const uint32_t xe_remote = map_to_cta(smem_u32(x_empty), peer);
    int64_t g = 0, pv_waited = 0;
    int seg = 0;
    int64_t u = u0;
    int k = u0 < u1 ? find_block(p.prefix, p.nblocks, u0) : 0;
    bool ok = true;
    while (u < u1 && ok) {
      const int64_t bstart = p.prefix[k], bend = p.prefix[k + 1];
      const int64_t send = u1 < bend ? u1 : bend;
      const int tile0 = (int)(u - bstart), ntl = (int)(send - u);
      const bool complete = (u == bstart) && (send == bend);
      const int b = k / p.nbps, rb = k % p.nbps;
      int64_t sstart; int T;
      seq_bounds(p, b, sstart, T);
      const int ri = rb * DEC_ROWS + row;
      const bool valid = ri < p.n_q * p.H;
      int cnt = 0;
      if (valid) {
        cnt = T;
        if (p.causal) {
          cnt = T - p.n_q + ri / p.H + 1;
          cnt = cnt < 0 ? 0 : (cnt > T ? T : cnt);
        }
      }
      float m_ref = -INFINITY, l = 0.f;
      for (int tt = 0; tt < ntl; ++tt, ++g) {
        const int sl = (int)(g & 1);
        const int use = (int)(g >> 1);
        if (*abort_flag || !mbar_wait(&s_full[sl], use & 1, p.wait_ns, p.status)) { ok = false; break; }
        tc_fence_after();
        float s[DEC_BT];
        {
          uint32_t r[32];
          tmem_ld32(tS + lane_off + sl * 64, r);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(r[c]);
          tmem_ld32(tS + lane_off + sl * 64 + 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) s[32 + c] = __uint_as_float(r[c]);
        }
        // exchange the partial scores with the peer CTA (16-byte chunks, XOR-swizzled by row)
        if (use >= 1 && !mbar_wait_cluster(&x_empty[sl], (use - 1) & 1, p.wait_ns, p.status)) { ok = false; break; }
        const uint32_t xrow_r = x_remote + (uint32_t)(sl * Cfg::X_SLOT + row * DEC_BT * 4);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint32_t chunk = (uint32_t)(c ^ (row & 7));
          st_cluster_v4(xrow_r + chunk * 16, s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
        }
        mbar_arrive_remote(xf_remote + sl * 8);
        if (!mbar_wait_cluster(&x_full[sl], use & 1, p.wait_ns, p.status)) { ok = false; break; }
        {
          const float4* xr = reinterpret_cast<const float4*>(sX + sl * (Cfg::X_SLOT / 4) + row * DEC_BT);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float4 v = xr[c ^ (row & 7)];
            s[4 * c] += v.x;
            s[4 * c + 1] += v.y;
            s[4 * c + 2] += v.z;
            s[4 * c + 3] += v.w;
          }
        }
        mbar_arrive_remote(xe_remote + sl * 8);
        // scale (log2 domain), mask, running maximum
        const int t0 = (tile0 + tt) * DEC_BT;
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < DEC_BT; ++c) {
          const float v = (t0 + c < cnt) ? s[c] * p.scale_log2 : -INFINITY;
          s[c] = v;
          mx = fmaxf(mx, v);
        }
        bool need = false;
        float factor = 1.f;
        if (mx > m_ref + 8.f) {
          if (m_ref != -INFINITY) {
            need = true;
            factor = ex2(m_ref - mx);
            l *= factor;
          }
          m_ref = mx;
        }
        const float mu = m_ref == -INFINITY ? 0.f : m_ref;
        float sum = 0.f;
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float p0 = ex2(s[2 * c] - mu), p1 = ex2(s[2 * c + 1] - mu);
          sum += p0 + p1;
          __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
          pk[c] = *reinterpret_cast<uint32_t*>(&h);
        }
        l += sum;
        tmem_st32(tS + lane_off + sl * 64, pk);
        tmem_wait_st();
        // the previous tile's P.C must be done before O is touched and before this P is released
        if (g > pv_waited) {
          if (!mbar_wait(o_done, (int)((g - 1) & 1), p.wait_ns, p.status)) { ok = false; break; }
          pv_waited = g;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll 1
          for (int cc = 0; cc < DEC_HALF; cc += 32) {
            uint32_t r[32];
            tmem_ld32(tO + lane_off + cc, r);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * factor);
            tmem_st32(tO + lane_off + cc, r);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(&p_full[sl]);
      }
      if (!ok) break;
      // epilogue of the segment: wait for its last P.C, then read this CTA's half of O
      if (g > pv_waited) {
        if (!mbar_wait(o_done, (int)((g - 1) & 1), p.wait_ns, p.status)) { ok = false; break; }
        pv_waited = g;
      }
      tc_fence_after();
      const int64_t orow = (int64_t)b * p.n_q * p.H + ri;
      const int slot = 2 * pair + (seg == 0 ? 0 : 1);
      const float inv = l > 0.f ? 1.f / l : 0.f;
      float* dst = complete ? p.out_lat + orow * DEC_DC + dim0
                            : p.o_part + ((int64_t)slot * DEC_ROWS + row) * DEC_DC + dim0;
      const float mul = complete ? inv : 1.f;
      const bool write = complete ? valid : true;
#pragma unroll 1
      for (int cc = 0; cc < DEC_HALF; cc += 32) {
        uint32_t r[32];
        tmem_ld32(tO + lane_off + cc, r);
        tmem_wait_ld();
        if (write) {
          float4* d4 = reinterpret_cast<float4*>(dst + cc);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            d4[c] = make_float4(__uint_as_float(r[4 * c]) * mul, __uint_as_float(r[4 * c + 1]) * mul,
                                __uint_as_float(r[4 * c + 2]) * mul, __uint_as_float(r[4 * c + 3]) * mul);
        }
      }
      if (rank == 0) {
        if (complete) {
          if (valid && p.lse) p.lse[orow] = l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
        } else {
          p.m_part[(int64_t)slot * DEC_ROWS + row] = m_ref;
          p.l_part[(int64_t)slot * DEC_ROWS + row] = l;
        }
      }
      tc_fence_before();
      u = send;
      ++seg;
      if (u < u1) k = find_block(p.prefix, p.nblocks, u);
    }
    if (!ok) *abort_flag = 1;
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();     // the peer may write into this CTA's exchange buffer until it is done
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------------------
// combine: one CTA per block; merges the partials of blocks split across clusters and writes
// zeros / -inf for blocks with nothing to attend to
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) decode_combine_tc_kernel(DecParams p) {
  const int k = blockIdx.x;
  const int64_t bstart = p.prefix[k], bend = p.prefix[k + 1];
  const int b = k / p.nbps, rb = k % p.nbps;
  const int rows_seq = p.n_q * p.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (bend == bstart) {
    for (int r = warp; r < DEC_ROWS; r += 8) {
      const int ri = rb * DEC_ROWS + r;
      if (ri >= rows_seq) break;
      const int64_t orow = (int64_t)b * rows_seq + ri;
      for (int d = lane; d < DEC_DC; d += 32) p.out_lat[orow * DEC_DC + d] = 0.f;
      if (lane == 0 && p.lse) p.lse[orow] = -INFINITY;
    }
    return;
  }
  const int64_t U = p.prefix[p.nblocks];
  const int p0 = find_owner(U, p.G, bstart), p1 = find_owner(U, p.G, bend - 1);
  if (p0 == p1) return;   // written whole by one cluster
  for (int r = warp; r < DEC_ROWS; r += 8) {
    const int ri = rb * DEC_ROWS + r;
    if (ri >= rows_seq) break;
    float M = -INFINITY;
    for (int q = p0; q <= p1; ++q) {
      const int slot = (q == p0 && bstart > range_start(U, p.G, q)) ? 2 * q + 1 : 2 * q;
      M = fmaxf(M, p.m_part[(int64_t)slot * DEC_ROWS + r]);
    }
    float L = 0.f;
    for (int q = p0; q <= p1; ++q) {
      const int slot = (q == p0 && bstart > range_start(U, p.G, q)) ? 2 * q + 1 : 2 * q;
      const float m = p.m_part[(int64_t)slot * DEC_ROWS + r];
      if (m != -INFINITY) L += ex2(m - M) * p.l_part[(int64_t)slot * DEC_ROWS + r];
    }
    const int64_t orow = (int64_t)b * rows_seq + ri;
    const float inv = L > 0.f ? 1.f / L : 0.f;
    for (int d = lane; d < DEC_DC; d += 32) {
      float acc = 0.f;
      for (int q = p0; q <= p1; ++q) {
        const int slot = (q == p0 && bstart > range_start(U, p.G, q)) ? 2 * q + 1 : 2 * q;
        const float m = p.m_part[(int64_t)slot * DEC_ROWS + r];
        if (m != -INFINITY) acc += ex2(m - M) * p.o_part[((int64_t)slot * DEC_ROWS + r) * DEC_DC + d];
      }
      p.out_lat[orow * DEC_DC + d] = acc * inv;
    }
    if (lane == 0 && p.lse) p.lse[orow] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
  }
}

// ---------------------------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------------------------
static int g_decode_clusters_override = 0;

void set_decode_clusters(int n) { g_decode_clusters_override = n > 0 ? n : 0; }

bool tc_decode_supported(const DecodeArgs& a) {
  return a.dc == DEC_DC && (a.dr == 0 || a.dr == 64) && a.H > 0 && a.n_q > 0 && a.total_rows > 0 &&
         (int64_t)a.batch * a.n_q * a.H < (1LL << 31) - DEC_ROWS && a.total_rows < (1LL << 31) - DEC_BT;
}

struct TcDecodePlan {
  int nbps, nblocks, G;
  size_t off_prefix, off_o, off_m, off_l, total;
};

static TcDecodePlan plan_tc(const DecodeArgs& a) {
  TcDecodePlan t;
  t.nbps = (int)ceil_div((int64_t)a.n_q * a.H, DEC_ROWS);
  t.nblocks = a.batch * t.nbps;
  const int64_t units_max = (int64_t)t.nblocks * std::max<int64_t>(1, ceil_div(a.max_seqlen, DEC_BT));
  int G = sm_count() / 2;
  if (g_decode_clusters_override > 0) G = g_decode_clusters_override;
  G = (int)std::max<int64_t>(1, std::min<int64_t>(G, units_max));
  t.G = G;
  t.off_prefix = 0;
  t.off_o = round_up((size_t)(t.nblocks + 1) * sizeof(int32_t), 256);
  t.off_m = t.off_o + (size_t)2 * G * DEC_ROWS * DEC_DC * sizeof(float);
  t.off_l = t.off_m + round_up((size_t)2 * G * DEC_ROWS * sizeof(float), 256);
  t.total = t.off_l + round_up((size_t)2 * G * DEC_ROWS * sizeof(float), 256);
  return t;
}

size_t tc_decode_workspace(const DecodeArgs& a) { return plan_tc(a).total; }

template <int DR>
static int launch_decode_t(const CUtensorMap& tq, const CUtensorMap& tk, const DecParams& p, cudaStream_t s) {
  static bool attr_set[64] = {false};
  const int dev = current_device();
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(tc_decode_kernel<DR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DecCfg<DR>::SMEM) != cudaSuccess)
      return MLA_ERR_CUDA;
    attr_set[dev] = true;
  }
  tc_decode_kernel<DR><<<2 * p.G, DEC_THREADS, DecCfg<DR>::SMEM, s>>>(tq, tk, p);
  MLA_LAUNCH_CHECK();
  return MLA_OK;
}

int tc_decode_launch(const DecodeArgs& a, cudaStream_t s) {
  const TcDecodePlan t = plan_tc(a);
  const int W = a.dc + a.dr;
  char* ws = static_cast<char*>(a.workspace);
  DecParams p{};
  p.cu = a.cu_seqlens; p.batch = a.batch; p.n_q = a.n_q; p.H = a.H; p.nbps = t.nbps; p.nblocks = t.nblocks;
  p.total_rows = a.total_rows; p.causal = a.causal ? 1 : 0;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.prefix = reinterpret_cast<int32_t*>(ws + t.off_prefix);
  p.G = t.G;
  p.out_lat = a.out_lat; p.lse = a.lse;
  p.o_part = reinterpret_cast<float*>(ws + t.off_o);
  p.m_part = reinterpret_cast<float*>(ws + t.off_m);
  p.l_part = reinterpret_cast<float*>(ws + t.off_l);
  p.status = device_status_ptr();
  p.wait_ns = (unsigned long long)wait_limit();
  if (!p.status) return MLA_ERR_CUDA;
  if (t.nblocks == 0) return MLA_OK;

  CUtensorMap tq, tk;
  {
    const uint64_t dims[2] = {(uint64_t)W, (uint64_t)a.batch * a.n_q * a.H};
    const uint64_t st[1] = {(uint64_t)W * 2};
    const uint32_t box[2] = {64, DEC_ROWS};
    if (!encode_tmap_bf16(&tq, const_cast<void*>(a.q_abs), 2, dims, st, box)) return MLA_ERR_CUDA;
  }
  {
    const uint64_t rows = (uint64_t)std::max<int64_t>(a.total_rows, 1);
    const uint64_t dims[2] = {(uint64_t)W, rows};
    const uint64_t st[1] = {(uint64_t)W * 2};
    const uint32_t box[2] = {64, DEC_BT};
    if (!encode_tmap_bf16(&tk, const_cast<void*>(a.cache), 2, dims, st, box)) return MLA_ERR_CUDA;
  }
  decode_plan_kernel<<<1, 1024, 0, s>>>(p, const_cast<int32_t*>(p.prefix));
  MLA_LAUNCH_CHECK();
  int st = a.dr == 0 ? launch_decode_t<0>(tq, tk, p, s) : launch_decode_t<64>(tq, tk, p, s);
  if (st) return st;
  decode_combine_tc_kernel<<<t.nblocks, 256, 0, s>>>(p);
  MLA_LAUNCH_CHECK();
  return MLA_OK;
}

}  // namespace mla
