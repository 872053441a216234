// tc_prefill.cu -- attention of un-absorbed heads over a whole prompt (prefill) on sm_100a.
//
// The un-absorbed form of the attention ("preacher-1/MLA_tutorial formula.md", Part 3, the
// training-form equation; "Gated MLA" (tensortonic), the problem equations: Q = X Wq^T, K = C Wk^T,
// V = C Wv^T, heads of D_h = D / H, causal mask, O = softmax(Q K^T / sqrt(D_h)) V): with every query
// of a prompt present, each head's keys and values are materialised once and attention runs on
// D_h-wide heads rather than on the d_c-wide absorbed ones, four times fewer multiply-adds per
// score and per output at the pages' widths ("formula.md", Part 3, the note after the inference
// form: the absorbed head is 4x wider; prefill is the compute-bound phase).
//
// One CTA = one (sequence, head, 128-query tile). Per 128-key tile j:
//   S_j = Q K_j^T          tcgen05, A = Q and B = K_j from shared memory (K-major), fp32 in TMEM
//   P_j = exp2(S_j * scale * log2(e) - m_ref), rows masked by the causal rule and the sequence end,
//         rounded to bf16 and written back to TMEM by the four softmax warps (one row per thread)
//   O  += P_j V_j          tcgen05, A = P_j from TMEM, B = V_j from shared memory (MN-major)
// S and P are double-buffered in TMEM (2 x 128 + 2 x 64 columns) next to O (128 columns), so the MMAs
// of S_{j+1} run while the softmax of j does. The reference maximum m_ref of a row moves only when a
// tile's maximum exceeds it by more than 8 (log2 units): P then stays below 2^8, and O and the row sum
// l, kept relative to the same m_ref, are rescaled together (after the pending P V products are
// done). Epilogue: O / l (times the optional gate), bf16. Tiles with more keys start first.
#include <cudaTypedefs.h>

#include <algorithm>

#include "sm100.cuh"
#include "tc.cuh"

namespace mla {

using namespace sm100;

constexpr int PF_BM = 128;                 // queries per CTA (the MMA's M)
constexpr int PF_BN = 128;                 // keys per tile (N of Q K^T, K of P V)
constexpr int PF_D = 128;                  // head width (K of Q K^T, N of P V)
constexpr int PF_THREADS = 384;            // warps 0 TMA, 1 MMA, 2-3 spare, 4-11 softmax (two per row window)
constexpr int PF_TILE = PF_BM * PF_D * 2;  // 32 KB: one Q, K or V tile, two 64-column boxes
constexpr int PF_BOX = PF_TILE / 2;        // 16 KB: one 128-row x 64-column box
constexpr int PF_SMEM = 5 * PF_TILE + 1024 + 4096;
constexpr uint32_t PF_TMEM_COLS = 512;
constexpr float PF_REF_SLACK = 8.f;        // log2 units a row maximum may exceed m_ref before it moves

__device__ __forceinline__ float pf_ex2(float x) {   // 2^x on the special-function unit (flushes tiny results)
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct PfParams {
  int B, S, H, n_qt;
  float scale_log2;                        // softmax scale times log2(e)
  int causal;
  const __nv_bfloat16* gate;               // [B*S, H*D] or null
  __nv_bfloat16* out;                      // [B*S, H*D]
  int* status;
  unsigned long long wait_ns;
};

struct PfBars {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], s_free[2], p_full[2], p_free[2];
  uint64_t done;                           // the MMA issuer's last commit
  uint32_t tmem;
  int abort;
  int last_k[2], last_v[2];                // the last tile loaded into each stage (abort drain)
  float xmax[2][2][PF_BM];                 // [tile parity][column half][row]: the halves' row maxima
  float xl[2][PF_BM];                      // [column half][row]: the halves' row sums
};

static_assert(sizeof(PfBars) <= 4096, "barrier region");

__global__ void __launch_bounds__(PF_THREADS, 1)
    tc_prefill_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv, PfParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + PF_TILE;            // [2] tiles
  uint8_t* sV = smem + 3 * PF_TILE;        // [2] tiles
  PfBars* bars = reinterpret_cast<PfBars*>(smem + 5 * PF_TILE);
  volatile int* abort_flag = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = p.B * p.H;
  const int qt = p.n_qt - 1 - (int)(blockIdx.x / BH);      // the longest rows of keys first
  const int bh = (int)(blockIdx.x % BH);
  const int b = bh / p.H, h = bh % p.H;
  const int q0 = qt * PF_BM;                                // first query of the tile, in its sequence
  const int row0 = b * p.S;                                 // the sequence's first row
  const int n_kt = (p.S + PF_BN - 1) / PF_BN;
  const int nkv = p.causal ? min(qt + 1, n_kt) : n_kt;      // key tiles this query tile reads

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], 8);
      mbar_init(&bars->p_full[i], 8);
      mbar_init(&bars->p_free[i], 1);
      bars->last_k[i] = -1;
      bars->last_v[i] = -1;
    }
    mbar_init(&bars->done, 1);
    bars->abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tq);
    prefetch_tmap(&tk);
    prefetch_tmap(&tv);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem, PF_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();                          // Q, K, V (and the gate) come from the previous kernels
  griddep_launch_dependents();
  const uint32_t tmem = bars->tmem;
  const uint32_t tS = tmem;                // [2] x 128 columns: scores
  const uint32_t tP = tmem + 256;          // [2] x 64 columns: bf16 probabilities (pairs)
  const uint32_t tO = tmem + 384;          // 128 columns: the output accumulator

  // a wait that gives up marks the CTA aborted; later waits of the CTA return false at once
  auto wait_bar = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity, p.wait_ns, p.status)) return true;
    *abort_flag = 1;
    return false;
  };
  // the same wait by every lane of a warp, with one outcome for all (the tensor-memory loads and
  // stores that follow are warp-collective)
  auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    const bool r = wait_bar(bar, parity);
    return __all_sync(0xffffffffu, r);
  };

  if (warp == 0 && lane == 0) {
    // ------------------------------- TMA producer -------------------------------
    // Q once; K_j and V_j into stage j & 1 once the MMAs of tile j - 2 have released it. Rows past the
    // last one of the tensors read as zeros; rows of the next sequence are masked or not stored.
    const int xh = h * PF_D;
    mbar_arrive_expect_tx(&bars->q_full, PF_TILE);
    tma_load_2d(sQ, &tq, &bars->q_full, xh, row0 + q0);
    tma_load_2d(sQ + PF_BOX, &tq, &bars->q_full, xh + 64, row0 + q0);
    for (int j = 0; j < nkv; ++j) {
      const int s = j & 1;
      const int y = row0 + j * PF_BN;
      if (j >= 2 && !wait_bar(&bars->k_empty[s], (uint32_t)((j >> 1) - 1) & 1u)) break;
      mbar_arrive_expect_tx(&bars->k_full[s], PF_TILE);
      tma_load_2d(sK + s * PF_TILE, &tk, &bars->k_full[s], xh, y);
      tma_load_2d(sK + s * PF_TILE + PF_BOX, &tk, &bars->k_full[s], xh + 64, y);
      bars->last_k[s] = j;
      if (j >= 2 && !wait_bar(&bars->v_empty[s], (uint32_t)((j >> 1) - 1) & 1u)) break;
      mbar_arrive_expect_tx(&bars->v_full[s], PF_TILE);
      tma_load_2d(sV + s * PF_TILE, &tv, &bars->v_full[s], xh, y);
      tma_load_2d(sV + s * PF_TILE + PF_BOX, &tv, &bars->v_full[s], xh + 64, y);
      bars->last_v[s] = j;
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------- MMA issuer -------------------------------
    // S_{j+1} = Q K_{j+1}^T is issued before O += P_j V_j, so it runs during the softmax of tile j
    constexpr uint32_t idesc_s = idesc_bf16_f32(PF_BM, PF_BN, false, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(PF_BM, PF_D, false, true);
    const uint32_t q_addr = smem_u32(sQ);
    auto issue_s = [&](int j) -> bool {
      const int s = j & 1;
      if (!wait_bar(&bars->k_full[s], (uint32_t)(j >> 1) & 1u)) return false;
      if (j >= 2 && !wait_bar(&bars->s_free[s], (uint32_t)((j >> 1) - 1) & 1u)) return false;
      tc_fence_after();
      const uint32_t k_addr = smem_u32(sK + s * PF_TILE);
#pragma unroll
      for (int kk = 0; kk < PF_D / 16; ++kk) {
        // K-major operands: 16 columns of the head width = 32 bytes along a swizzled 128-byte row;
        // columns 64.. are in the second box
        const uint32_t off = (uint32_t)((kk >> 2) * PF_BOX + (kk & 3) * 32);
        mma_bf16_ss(tS + s * PF_BN, smem_desc_sw128(q_addr + off, 16, 1024), smem_desc_sw128(k_addr + off, 16, 1024),
                    idesc_s, kk > 0 ? 1u : 0u);
      }
      mma_commit(&bars->k_empty[s]);
      mma_commit(&bars->s_full[s]);
      return true;
    };
    auto issue_pv = [&](int j) -> bool {
      const int s = j & 1;
      if (!wait_bar(&bars->p_full[s], (uint32_t)(j >> 1) & 1u)) return false;
      if (!wait_bar(&bars->v_full[s], (uint32_t)(j >> 1) & 1u)) return false;
      tc_fence_after();
      const uint32_t v_addr = smem_u32(sV + s * PF_TILE);
#pragma unroll
      for (int kk = 0; kk < PF_BN / 16; ++kk)
        // A = 16 keys of P (8 TMEM columns of bf16 pairs); B = the same 16 keys of V, MN-major: rows of
        // 64 head columns, 8-key groups 1024 bytes apart, the two 64-column boxes PF_BOX apart
        mma_bf16_ts(tO, tP + s * 64 + kk * 8, smem_desc_sw128(v_addr + kk * 2048, PF_BOX, 1024), idesc_o,
                    (j > 0 || kk > 0) ? 1u : 0u);
      mma_commit(&bars->v_empty[s]);
      mma_commit(&bars->p_free[s]);    // also: O holds every product up to P_j V_j
      return true;
    };
    bool ok = wait_bar(&bars->q_full, 0);
    if (ok) ok = issue_s(0);
    for (int j = 0; ok && j < nkv; ++j) {
      if (j + 1 < nkv) ok = issue_s(j + 1);
      if (ok) ok = issue_pv(j);
    }
    mma_commit(&bars->done);
  } else if (warp >= 4) {
    // ------------------------------- softmax and epilogue -------------------------------
    // Two warps per TMEM lane window: warp 4 + q takes key columns 0-63 of rows 32 q .., warp 8 + q
    // columns 64-127 (and the matching halves of O). The pair shares its rows' maxima and sums through
    // shared memory at a 64-thread named barrier that also carries an abort decision, so that both
    // warps of a pair always take the same path.
    const int quarter = warp & 3;                  // TMEM lanes 32 quarter .. (the warp's lane window)
    const int half = (warp - 4) >> 2;              // key / head columns [64 half, 64 half + 64)
    const uint32_t bar_id = 1 + (uint32_t)quarter;
    const int row = quarter * 32 + lane;           // query row of the tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int qi = q0 + row;                       // query position in its sequence
    const int k_end = min(p.S, p.causal ? qi + 1 : p.S);   // keys 0 .. k_end - 1 are visible
    float m_ref = 0.f, l = 0.f;
    bool alive = true;                             // this warp's waits have all succeeded
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int s = j & 1;
      const bool okj = alive && warp_wait(&bars->s_full[s], (uint32_t)(j >> 1) & 1u);
      uint32_t xr[PF_BN / 2];
      float mh = -INFINITY;
      if (okj) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c)
          tmem_ld32(tS + s * PF_BN + lane_off + half * 64 + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&xr[32 * c]));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free[s]);
        const int kmax = k_end - j * PF_BN - half * 64;
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // four independent chains
#pragma unroll
        for (int c = 0; c < PF_BN / 2; ++c) {
          const float v = c < kmax ? __uint_as_float(xr[c]) * p.scale_log2 : -INFINITY;
          xr[c] = __float_as_uint(v);
          mx[c & 3] = fmaxf(mx[c & 3], v);
        }
        mh = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        bars->xmax[j & 1][half][row] = mh;
      }
      if (named_bar_or(bar_id, 64, !okj)) { ok = false; break; }
      const float mt = fmaxf(bars->xmax[j & 1][0][row], bars->xmax[j & 1][1][row]);
      // P buffer s is free once P_{j-2} V_{j-2} is done
      if (j >= 2 && !warp_wait(&bars->p_free[s], (uint32_t)((j >> 1) - 1) & 1u)) { alive = false; continue; }
      if (j == 0) {
        m_ref = mt == -INFINITY ? 0.f : mt;
      } else {
        const bool move = mt > m_ref + PF_REF_SLACK;
        if (__any_sync(0xffffffffu, move)) {
          // O (every product up to P_{j-1} V_{j-1}, done once p_free of tile j - 1 completes) and l
          // follow the rows' new reference maxima (this warp's half of O); the other rows keep theirs
          const int sp = (j - 1) & 1;
          if (!warp_wait(&bars->p_free[sp], (uint32_t)((j - 1) >> 1) & 1u)) { alive = false; continue; }
          tc_fence_after();
          const float f = move ? pf_ex2(m_ref - mt) : 1.f;
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + lane_off + half * 64 + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * f);
            tmem_st32(tO + lane_off + half * 64 + c * 32, r);
          }
          tmem_wait_st();
          if (move) {
            l *= f;
            m_ref = mt;
          }
        }
      }
      // probabilities, rounded to bf16 once; the row sum adds the rounded values the MMA will use
      uint32_t pk[PF_BN / 4];
      float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < PF_BN / 4; ++c) {
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(pf_ex2(__uint_as_float(xr[2 * c]) - m_ref),
                                                        pf_ex2(__uint_as_float(xr[2 * c + 1]) - m_ref));
        const float2 back = __bfloat1622float2(b2);
        rs[c & 3] += back.x + back.y;
        pk[c] = *reinterpret_cast<const uint32_t*>(&b2);
      }
      l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
      tc_fence_after();
      tmem_st32(tP + s * 64 + lane_off + half * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[s]);
    }
    // epilogue: O / l (times the gate), bf16, once the last P V product is done; l is the sum of the
    // pair's two halves, added in a fixed order
    bool okf = ok && alive;
    if (okf && nkv > 0) okf = warp_wait(&bars->p_free[(nkv - 1) & 1], (uint32_t)((nkv - 1) >> 1) & 1u);
    if (ok) {
      bars->xl[half][row] = l;
      const bool bad = named_bar_or(bar_id, 64, !okf);
      if (!bad) {
        tc_fence_after();
        const float lt = bars->xl[0][row] + bars->xl[1][row];
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const bool store = qi < p.S;
        const int64_t ld = (int64_t)p.H * PF_D;
        __nv_bfloat16* dst = p.out + (int64_t)(row0 + qi) * ld + h * PF_D + half * 64;
        const __nv_bfloat16* g = p.gate ? p.gate + (int64_t)(row0 + qi) * ld + h * PF_D + half * 64 : nullptr;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + lane_off + half * 64 + c * 32, r);
          tmem_wait_ld();
          if (!store) continue;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(r[8 * q + e]) * inv;
            if (g) {
              const uint4 gv = *reinterpret_cast<const uint4*>(g + c * 32 + 8 * q);
              const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 gf = __bfloat1622float2(g2[e]);
                v[2 * e] *= gf.x;
                v[2 * e + 1] *= gf.y;
              }
            }
            uint4 w;
            uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 o2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
              wp[e] = *reinterpret_cast<const uint32_t*>(&o2);
            }
            *reinterpret_cast<uint4*>(dst + c * 32 + 8 * q) = w;
          }
        }
      }
    }
  }

  // ---- teardown: nothing of this CTA's may be in flight when its tensor memory is released ----
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t drain_ns = p.wait_ns > 100000000ull ? p.wait_ns : 100000000ull;
    if (*abort_flag) {
      // only the last load of a stage can be in flight (a later one waited for the MMAs to read it)
      for (int s = 0; s < 2; ++s) {
        if (bars->last_k[s] >= 0) (void)mbar_wait(&bars->k_full[s], (uint32_t)(bars->last_k[s] >> 1) & 1u, drain_ns, p.status);
        if (bars->last_v[s] >= 0) (void)mbar_wait(&bars->v_full[s], (uint32_t)(bars->last_v[s] >> 1) & 1u, drain_ns, p.status);
      }
    }
    (void)mbar_wait(&bars->done, 0, drain_ns, p.status);   // the MMA issuer's final commit
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, PF_TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------------------------
bool tc_prefill_supported(int64_t B, int64_t S, int64_t H, int64_t D) {
  return D == PF_D && B > 0 && S > 0 && H > 0 && B * S < (1LL << 31) - PF_BN && B * H * ((S + PF_BM - 1) / PF_BM) <
         (1LL << 31) && H * D < (1LL << 24);
}

int tc_prefill_launch(const void* q, const void* k, const void* v, const void* gate, int64_t B, int64_t S, int64_t H,
                      float scale, bool causal, void* out, cudaStream_t s) {
  static bool attr_set[64] = {false};
  const int dev = current_device();
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(tc_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PF_SMEM) != cudaSuccess)
      return MLA_ERR_CUDA;
    attr_set[dev] = true;
  }
  // Q, K, V: [B*S rows][H*D columns] bf16; boxes of 64 columns x 128 rows
  CUtensorMap tq, tk, tv;
  const uint64_t dims[2] = {(uint64_t)(H * PF_D), (uint64_t)(B * S)};
  const uint64_t st[1] = {(uint64_t)(H * PF_D * 2)};
  const uint32_t box[2] = {64, 128};
  if (!encode_tmap_bf16(&tq, const_cast<void*>(q), 2, dims, st, box) ||
      !encode_tmap_bf16(&tk, const_cast<void*>(k), 2, dims, st, box) ||
      !encode_tmap_bf16(&tv, const_cast<void*>(v), 2, dims, st, box))
    return MLA_ERR_CUDA;
  PfParams p{};
  p.B = (int)B; p.S = (int)S; p.H = (int)H; p.n_qt = (int)((S + PF_BM - 1) / PF_BM);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  p.gate = static_cast<const __nv_bfloat16*>(gate);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.status = device_status_ptr();
  p.wait_ns = (unsigned long long)wait_limit();
  if (!p.status) return MLA_ERR_CUDA;
  const int64_t grid = B * H * p.n_qt;
  return launch_pdl(tc_prefill_kernel, dim3((unsigned)grid), dim3(PF_THREADS), (size_t)PF_SMEM, s, tq, tk, tv, p);
}

}  // namespace mla
