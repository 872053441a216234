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
//  * O (128 rows x 512 latent columns, fp32) fills the 512 columns of one SM's tensor memory, so a
//    CLUSTER OF TWO CTAs shares a block, with different jobs:
//      - the score CTA (rank 0) holds the block's latent query in TMEM (256 columns of bf16 pairs, the
//        A operand of QK^T) and its rotary query in shared memory, streams every cache row whole (all
//        576 columns, 128-position tiles by TMA), computes S = Q K^T in fp32 into one of two 128-column
//        TMEM slots, runs the online softmax in fp32 and hands P (bf16) to the value CTA through
//        distributed shared memory, 64 positions at a time, with per-row side data (the factor by
//        which O must be rescaled, and at the end of a block the row maximum and sum);
//      - the value CTA (rank 1) holds all of O in TMEM, streams the latent columns of the same rows
//        (read a second time, from L2, right after the score CTA brought them in) and accumulates
//        O += P . C with 128 x 256 x 16 MMAs, rescales O rows when told to, and writes the result.
//    The scores never leave the score CTA, and they are never rounded below fp32 before the
//    exponential: the hand-over is one-way (P and side data forward, "slot free" back).
//  * The score CTA rescales nothing: P is taken against a reference maximum that moves only when a
//    row's maximum grows by more than 2^8 (exact: numerator and denominator share it); the rare move
//    is passed on with the P of that tile, and the value CTA multiplies its O rows before that P.C.
//  * Work: the (block, 128-position tile) units of all sequences are split evenly over the clusters
//    (persistent). A cluster that covers a whole block writes the normalised result; split blocks
//    leave (O, max, sum) partials that a combine kernel merges.
//  * Warp roles (384 threads). Score CTA: warp 0 lane 0 TMA, warp 1 lane 0 QK^T, warps 4-11 softmax
//    (warp w: rows 32 (w & 3) .., positions [64 h, 64 h + 64) of each tile, h = (w - 4) >> 2), which
//    also load each block's latent query into TMEM. Value CTA: warp 0 lane 0 TMA, warp 1 lane 0 P.C,
//    warp 2 lane 0 hands P slots back, warps 4-11 rescale and write O (warp w: rows 32 (w & 3) ..,
//    O columns [256 h, 256 h + 256)).
//  * Every wait is bounded (global-timer limit); a wait that gives up sets the library's status word,
//    and the CTA abandons its work: it issues nothing more, drains its own TMA loads, MMAs and bulk
//    copies and leaves through the cluster barrier.
#include <math.h>

#include <algorithm>

#include "sm100.cuh"
#include "tc.cuh"

namespace mla {

using namespace sm100;

constexpr int DEC_BT = 128;        // positions per score tile
constexpr int DEC_HT = 64;         // positions per P hand-over (half a tile)
constexpr int DEC_THREADS = 384;
constexpr int DEC_DC = 512;        // latent width handled by this kernel
constexpr int DEC_ROWS = 128;      // rows per block
constexpr int DEC_NPH = 3;         // P half-tile slots in the value CTA
constexpr float DEC_MOVE = 8.f;    // the reference maximum moves when a row maximum exceeds it by 2^8
constexpr int DEC_SMEM_LIMIT = 232448;   // dynamic shared memory per CTA (227 KB)
constexpr int DEC_BAR_BYTES = 1024;

__host__ __device__ constexpr int dec_round1024(int x) { return (x + 1023) / 1024 * 1024; }
__host__ __device__ constexpr int dec_max(int a, int b) { return a > b ? a : b; }

template <int DR>
struct DecCfg {
  static constexpr int DATA_LIMIT = DEC_SMEM_LIMIT - 1024 - DEC_BAR_BYTES;   // 1 KB for alignment
  static constexpr int NB = 8 + (DR ? 1 : 0);              // 64-column boxes of a cache row
  static constexpr int BOX = DEC_BT * 128;                 // 128 positions x 64 columns bf16: 16 KB
  // score CTA
  static constexpr int S_OFF_QR = 0;                       // rotary query [128 rows x 64 columns]
  static constexpr int S_QR = DR ? DEC_ROWS * 128 : 0;
  static constexpr int S_OFF_PS = S_OFF_QR + S_QR;         // P staging: 8 warps x 4 KB (32 rows x 128 B)
  static constexpr int S_OFF_SIDE = S_OFF_PS + 8 * 4096;   // side staging: 8 warps x 512 B
  static constexpr int S_OFF_RED = S_OFF_SIDE + 8 * 512;   // row maxima [2][2][128], row sums [128]
  static constexpr int S_OFF_K = dec_round1024(S_OFF_RED + 5 * DEC_ROWS * 4);
  static constexpr int NK = (DATA_LIMIT - S_OFF_K) / BOX;  // cache boxes in flight
  // value CTA
  static constexpr int PH = DEC_ROWS * 128;                // P of a half tile: 128 rows x 64 positions bf16
  static constexpr int SIDE = 4 * 512;                     // side data of a half tile: 4 quarters x 512 B
  static constexpr int PSLOT = PH + SIDE;                  // 18 KB (a multiple of 1024)
  static constexpr int V_OFF_P = 0;
  static constexpr int V_OFF_V = dec_round1024(DEC_NPH * PSLOT);
  static constexpr int UNIT = DEC_HT * 512;                // 64 positions x 256 latent columns bf16: 32 KB
  static constexpr int NV = (DATA_LIMIT - V_OFF_V) / UNIT; // value units in flight
  static constexpr int OFF_BAR = dec_max(S_OFF_K + NK * BOX, V_OFF_V + NV * UNIT);
  static constexpr int SMEM = OFF_BAR + DEC_BAR_BYTES + 1024;
  static_assert(PSLOT % 1024 == 0, "P slots must keep the 1024-byte swizzle alignment");
  static_assert(NK >= NB, "a whole tile of cache boxes must fit in the ring");
  static_assert(NV >= 2, "the value ring needs two units");
  static_assert(SMEM <= DEC_SMEM_LIMIT, "shared memory budget");
};

// side data of one warp's 32 rows for one half tile (512 B, the layout both CTAs use)
struct DecSide {
  int flag;          // some row of these 32 moved its reference maximum at this tile
  int pad[3];
  float alpha[32];   // factor for O of each row (1 where the reference did not move)
  float m[32];       // reference maximum (log2 units) after this tile
  float l[32];       // row sum after this tile (whole row at the last tile of a block)
  float pad2[28];
};
static_assert(sizeof(DecSide) == 512, "side record size");

template <int NK, int NV>
struct DecBars {
  // score CTA
  uint64_t k_full[NK], k_empty[NK];
  uint64_t qr_full, q_tm, q_empty;
  uint64_t s_full[2], s_empty[2];
  uint64_t p_empty[DEC_NPH];      // arrived by the value CTA: a P slot may be written again
  // value CTA
  uint64_t v_full[NV], v_empty[NV];
  uint64_t p_full[DEC_NPH];       // P + side data landed (transaction count of the bulk copies)
  uint64_t pfree[DEC_NPH];        // P.C read the slot and the rescale/epilogue warps read its side data
  uint64_t o_fix, fix_done;       // rescale hand-shake (one phase per rescale)
  uint64_t o_fin, o_free;         // epilogue hand-shake (one phase per block segment)
  // both
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort_flag;
};

struct DecParams {
  const __nv_bfloat16* q_abs;  // [q_rows][W]
  int64_t q_rows;
  int W;
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

// positions row ri (within its sequence's n_q * H rows) attends to
__device__ __forceinline__ int row_count(int T, int n_q, int H, int ri, int causal) {
  if (ri >= n_q * H) return 0;
  if (!causal) return T;
  const int c = T - n_q + ri / H + 1;
  return c < 0 ? 0 : (c > T ? T : c);
}

// tiles a block needs: up to the last position its last valid row sees
__device__ __forceinline__ int block_tiles(int T, int n_q, int H, int rb, int causal) {
  const int rows = n_q * H;
  const int last_row = min(rows - 1, rb * DEC_ROWS + DEC_ROWS - 1);
  const int cnt = row_count(T, n_q, H, last_row, causal);
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

// The segments of a cluster's unit range [u0, u1): the part of one block that the range covers.
struct DecSeg {
  int k;              // block
  int b, rb;          // sequence, row block within it
  int tile0, ntl;     // first tile of the block in this segment, tiles in it
  bool complete;      // the segment is the whole block
  int64_t sstart;     // first cache row of the sequence
  int T;              // sequence length
};

struct DecWalk {
  int64_t u, u1;
  int k;
  __device__ void begin(const DecParams& p, int64_t u0, int64_t u1_) {
    u = u0;
    u1 = u1_;
    k = u0 < u1 ? find_block(p.prefix, p.nblocks, u0) : 0;
  }
  __device__ bool next(const DecParams& p, DecSeg& s) {
    if (u >= u1) return false;
    const int64_t bstart = p.prefix[k], bend = p.prefix[k + 1];
    const int64_t send = u1 < bend ? u1 : bend;
    s.k = k;
    s.b = k / p.nbps;
    s.rb = k % p.nbps;
    s.tile0 = (int)(u - bstart);
    s.ntl = (int)(send - u);
    s.complete = (u == bstart) && (send == bend);
    seq_bounds(p, s.b, s.sstart, s.T);
    u = send;
    if (u < u1) k = find_block(p.prefix, p.nblocks, u);
    return true;
  }
};

// ---------------------------------------------------------------------------------------------
// plan: tiles per block and their exclusive prefix (one CTA)
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) decode_plan_kernel(DecParams p, int32_t* prefix) {
  __shared__ int64_t sums[1024];
  griddep_wait();                // cu_seqlens and the workspace may be in use by earlier work
  griddep_launch_dependents();
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
    tc_decode_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                     const __grid_constant__ CUtensorMap tqr, DecParams p) {
  using Cfg = DecCfg<DR>;
  constexpr int NK = Cfg::NK;
  constexpr int NV = Cfg::NV;
  constexpr int NB = Cfg::NB;
  constexpr int NPH = DEC_NPH;
  using Bars = DecBars<NK, NV>;
  static_assert(sizeof(Bars) <= DEC_BAR_BYTES, "barrier block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + Cfg::OFF_BAR);
  volatile int* abort_flag = &bars->abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const bool scorer = rank == 0;

  if (tid == 0) {
    if (scorer) {
      for (int s = 0; s < NK; ++s) {
        mbar_init(&bars->k_full[s], 1);
        mbar_init(&bars->k_empty[s], 1);
      }
      mbar_init(&bars->qr_full, 1);
      mbar_init(&bars->q_tm, 8);          // one arrival per softmax warp (each writes its share of Q)
      mbar_init(&bars->q_empty, 1);
      for (int s = 0; s < 2; ++s) {
        mbar_init(&bars->s_full[s], 1);
        mbar_init(&bars->s_empty[s], 8);  // every softmax warp has read its part of the slot
      }
      for (int s = 0; s < NPH; ++s) mbar_init(&bars->p_empty[s], 1);
    } else {
      for (int s = 0; s < NV; ++s) {
        mbar_init(&bars->v_full[s], 1);
        mbar_init(&bars->v_empty[s], 1);
      }
      for (int s = 0; s < NPH; ++s) {
        mbar_init(&bars->p_full[s], 1);
        mbar_init(&bars->pfree[s], 9);    // the P.C commit and the 8 rescale / epilogue warps
      }
      mbar_init(&bars->o_fix, 1);
      mbar_init(&bars->fix_done, 8);
      mbar_init(&bars->o_fin, 1);
      mbar_init(&bars->o_free, 8);
      // arm the first use of every P slot: one local arrival plus the score CTA's copies
      for (int s = 0; s < NPH; ++s) mbar_arrive_expect_tx(&bars->p_full[s], Cfg::PSLOT);
    }
    mbar_init(&bars->drain[0], 1);
    mbar_init(&bars->drain[1], 1);
    bars->abort_flag = 0;
    fence_mbar_init();
    if (scorer) {
      prefetch_tmap(&tk);
      if (DR) prefetch_tmap(&tqr);
    } else {
      prefetch_tmap(&tv);
    }
  }
  if (warp == 0) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();           // the peer's barriers are initialised before any remote access
  tc_fence_after();
  griddep_wait();           // the plan, the query block and the cache come from earlier kernels
  griddep_launch_dependents();
  const uint32_t tmem = bars->tmem_base;

  const int64_t U = p.prefix[p.nblocks];
  const int64_t u0 = range_start(U, p.G, pair), u1 = range_start(U, p.G, pair + 1);
  const int64_t drain_ns = p.wait_ns > 100000000ull ? p.wait_ns : 100000000ull;
  // a wait that gives up marks the CTA aborted; later waits of the CTA return false at once
  auto wait_bar = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity, p.wait_ns, p.status)) return true;
    *abort_flag = 1;
    return false;
  };

  if (scorer) {
    // =========================================================================================
    // score CTA
    // =========================================================================================
    const uint32_t tQ = tmem;            // columns [0, 256): latent query, bf16 pairs
    const uint32_t tS = tmem + 256;      // columns [256, 512): two 128-column S slots
    uint8_t* sQR = smem + Cfg::S_OFF_QR;
    uint8_t* sK = smem + Cfg::S_OFF_K;
    if (warp == 0 && lane == 0) {
      // ------------------------------- TMA producer -------------------------------
      DecWalk w;
      w.begin(p, u0, u1);
      DecSeg sg;
      int64_t n = 0;          // boxes issued
      int segi = 0, qr_loads = 0;
      bool ok = true;
      while (ok && w.next(p, sg)) {
        const int qrow = (int)((int64_t)sg.b * p.n_q * p.H + (int64_t)sg.rb * DEC_ROWS);
        for (int tt = 0; tt < sg.ntl && ok; ++tt) {
          const int y = (int)(sg.sstart + (int64_t)(sg.tile0 + tt) * DEC_BT);
          for (int j = 0; j < NB; ++j, ++n) {
            const int s = (int)(n % NK);
            if (n >= NK && !wait_bar(&bars->k_empty[s], (uint32_t)((n / NK) - 1) & 1u)) { ok = false; break; }
            mbar_arrive_expect_tx(&bars->k_full[s], Cfg::BOX);
            tma_load_2d(sK + s * Cfg::BOX, &tk, &bars->k_full[s], 64 * j, y);
          }
          if (!ok) break;
          if (DR && tt == 0) {
            // the rotary query of this segment, once the previous segment's last QK^T has read the old one
            if (segi > 0 && !wait_bar(&bars->q_empty, (uint32_t)(segi - 1) & 1u)) { ok = false; break; }
            mbar_arrive_expect_tx(&bars->qr_full, DEC_ROWS * 128);
            tma_load_2d(sQR, &tqr, &bars->qr_full, DEC_DC, qrow);
            ++qr_loads;
          }
        }
        ++segi;
      }
      if (*abort_flag) {
        // drain this CTA's own loads in flight before the shared memory is released
        for (int64_t i = (n > NK ? n - NK : 0); i < n; ++i)
          (void)mbar_wait(&bars->k_full[i % NK], (uint32_t)(i / NK) & 1u, drain_ns, p.status);
        if (qr_loads > 0) (void)mbar_wait(&bars->qr_full, (uint32_t)(qr_loads - 1) & 1u, drain_ns, p.status);
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------- QK^T issuer -------------------------------
      // S[slot] = Q K^T over the tile's 128 positions: latent boxes from the TMEM query (A) and the
      // cache box (B, K-major), the rotary box from the shared-memory query. Each cache box is released
      // by a commit as soon as its four MMAs complete.
      constexpr uint32_t idesc = idesc_bf16_f32(128, DEC_BT, false, false);
      const uint64_t kd0 = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t qd0 = smem_desc_sw128(smem_u32(sQR), 16, 1024);
      constexpr uint64_t kBox = (uint64_t)(Cfg::BOX >> 4);
      DecWalk w;
      w.begin(p, u0, u1);
      DecSeg sg;
      int64_t n = 0, g = 0;
      int segi = 0;
      bool ok = true;
      while (ok && w.next(p, sg)) {
        if (!wait_bar(&bars->q_tm, (uint32_t)segi & 1u)) { ok = false; break; }
        if (DR && !wait_bar(&bars->qr_full, (uint32_t)segi & 1u)) { ok = false; break; }
        for (int tt = 0; tt < sg.ntl; ++tt, ++g) {
          const int sl = (int)(g & 1);
          if (g >= 2 && !wait_bar(&bars->s_empty[sl], (uint32_t)((g >> 1) - 1) & 1u)) { ok = false; break; }
          tc_fence_after();
          const uint32_t td = tS + sl * DEC_BT;
          for (int j = 0; j < NB; ++j, ++n) {
            const int s = (int)(n % NK);
            if (!wait_bar(&bars->k_full[s], (uint32_t)(n / NK) & 1u)) { ok = false; break; }
            tc_fence_after();
            const uint64_t kd = kd0 + (uint64_t)s * kBox;
            if (j < 8) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ts(td, tQ + j * 32 + kk * 8, kd + (uint64_t)(kk * 2), idesc, (j | kk) ? 1u : 0u);
            } else {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(td, qd0 + (uint64_t)(kk * 2), kd + (uint64_t)(kk * 2), idesc, 1u);
            }
            mma_commit(&bars->k_empty[s]);
          }
          if (!ok) break;
          mma_commit(&bars->s_full[sl]);
          if (tt + 1 == sg.ntl) mma_commit(&bars->q_empty);
        }
        ++segi;
      }
      if (!ok || *abort_flag) {
        *abort_flag = 1;
        // every MMA this thread issued must finish before TMEM is released
        mma_commit(&bars->drain[0]);
        (void)mbar_wait(&bars->drain[0], 0, drain_ns, p.status);
      }
    } else if (warp >= 4) {
      // -------------------------------- softmax --------------------------------
      const int w8 = warp - 4, q = w8 & 3, hh = w8 >> 2;
      const int row = q * 32 + lane;
      const uint32_t lane_off = (uint32_t)(q * 32) << 16;
      uint8_t* stg = smem + Cfg::S_OFF_PS + hh * 16384 + q * 4096;   // this warp's 32 rows of P
      DecSide* side = reinterpret_cast<DecSide*>(smem + Cfg::S_OFF_SIDE + w8 * 512);
      float* red = reinterpret_cast<float*>(smem + Cfg::S_OFF_RED);  // [2 tiles][2 halves][128], then sums
      const uint32_t p_remote = map_to_cta(smem_u32(smem + Cfg::V_OFF_P), 1);
      const uint32_t pf_remote = map_to_cta(smem_u32(&bars->p_full[0]), 1);
      bool copies = false;    // this lane has bulk copies whose source reads may be pending
      DecWalk w;
      w.begin(p, u0, u1);
      DecSeg sg;
      int64_t g = 0;
      int segi = 0;
      while (w.next(p, sg)) {
        // ---- the block's latent query into TMEM: rows 32 q .., latent columns [256 hh, 256 hh + 256)
        if (segi > 0) (void)wait_bar(&bars->q_empty, (uint32_t)(segi - 1) & 1u);
        tc_fence_after();
        if (lane == 0 && copies) bulk_wait_read_all();   // the staging area is free again
        __syncwarp();
        {
          const int64_t qr0 = (int64_t)sg.b * p.n_q * p.H + (int64_t)sg.rb * DEC_ROWS + q * 32;
          const int chunk = lane & 7;
#pragma unroll 1
          for (int r4 = 0; r4 < 4; r4 += 2) {
            uint4 v[2][8];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int col0 = hh * 256 + (r4 + h2) * 64;
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int64_t qr = qr0 + 4 * j + (lane >> 3);
                const uint4* src = reinterpret_cast<const uint4*>(p.q_abs + qr * p.W + col0) + chunk;
                v[h2][j] = qr < p.q_rows ? *src : make_uint4(0u, 0u, 0u, 0u);
              }
            }
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int rr = 4 * j + (lane >> 3);
                *reinterpret_cast<uint4*>(stg + rr * 128 + ((chunk ^ (rr & 7)) * 16)) = v[h2][j];
              }
              __syncwarp();
              uint32_t r[32];
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const uint4 x = *reinterpret_cast<const uint4*>(stg + lane * 128 + ((c ^ (lane & 7)) * 16));
                r[4 * c] = x.x; r[4 * c + 1] = x.y; r[4 * c + 2] = x.z; r[4 * c + 3] = x.w;
              }
              __syncwarp();
              tmem_st32(tQ + lane_off + hh * 128 + (r4 + h2) * 32, r);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->q_tm);
        }
        const int cnt = row_count(sg.T, p.n_q, p.H, sg.rb * DEC_ROWS + row, p.causal);
        float m_ref = -INFINITY, l = 0.f;
        for (int tt = 0; tt < sg.ntl; ++tt, ++g) {
          const int sl = (int)(g & 1);
          const bool last = tt + 1 == sg.ntl;
          float s[64];
          (void)wait_bar(&bars->s_full[sl], (uint32_t)(g >> 1) & 1u);
          tc_fence_after();
          {
            uint32_t r0[32], r1[32];
            tmem_ld32(tS + lane_off + sl * DEC_BT + hh * 64, r0);
            tmem_ld32(tS + lane_off + sl * DEC_BT + hh * 64 + 32, r1);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              s[c] = __uint_as_float(r0[c]);
              s[32 + c] = __uint_as_float(r1[c]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0 && !*abort_flag) mbar_arrive(&bars->s_empty[sl]);
          // mask (only where the tile crosses the row's limit) and the raw row maximum
          const int t0 = (sg.tile0 + tt) * DEC_BT + hh * 64;
          if (t0 + 64 > cnt) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (t0 + c >= cnt) s[c] = -INFINITY;
          }
          float m4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
          for (int c = 4; c < 64; c += 4) {
            m4[0] = fmaxf(m4[0], s[c]);
            m4[1] = fmaxf(m4[1], s[c + 1]);
            m4[2] = fmaxf(m4[2], s[c + 2]);
            m4[3] = fmaxf(m4[3], s[c + 3]);
          }
          float* mx = red + (g & 1) * 2 * DEC_ROWS;
          mx[hh * DEC_ROWS + row] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
          named_bar_sync(1 + q, 64);          // the two warps of these rows
          const float mx_t = fmaxf(mx[row], mx[DEC_ROWS + row]) * p.scale_log2;   // the scale is positive
          float alpha = 1.f;
          bool moved = false;
          if (mx_t > m_ref + DEC_MOVE) {
            if (m_ref != -INFINITY) {
              alpha = ex2(m_ref - mx_t);
              moved = true;
              l *= alpha;
            }
            m_ref = mx_t;
          }
          const float mu = m_ref == -INFINITY ? 0.f : m_ref;
          // P in bf16 (round to nearest even), and the row sum of the same rounded values, so that
          // numerator and denominator of the normalisation share the rounding
          uint32_t pk[32];
          float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(ex2(fmaf(s[2 * c], p.scale_log2, -mu)),
                                                            ex2(fmaf(s[2 * c + 1], p.scale_log2, -mu)));
            pk[c] = *reinterpret_cast<const uint32_t*>(&b2);
            sum0 += __uint_as_float(pk[c] << 16);
            sum1 += __uint_as_float(pk[c] & 0xFFFF0000u);
          }
          l += sum0 + sum1;
          if (last) {
            // the block's row sum is the sum of both halves: the second warp of the pair sends it
            float* ls = red + 4 * DEC_ROWS;
            if (hh == 0) ls[row] = l;
            named_bar_sync(1 + q, 64);
            if (hh == 1) l += ls[row];
          }
          const int flag = (hh == 0) ? (__any_sync(0xffffffffu, moved) ? 1 : 0) : 0;
          // the P slot of this half tile must have been handed back by the value CTA
          const int64_t i = 2 * g + hh;
          const int hs = (int)(i % NPH);
          if (i >= NPH) (void)wait_bar(&bars->p_empty[hs], (uint32_t)((i / NPH) - 1) & 1u);
          if (lane == 0 && copies) bulk_wait_read_all();  // the previous copies have read the staging area
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(stg + lane * 128 + ((c ^ (lane & 7)) * 16)) =
                make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          if (lane == 0) side->flag = flag;
          side->alpha[lane] = hh == 0 ? alpha : 1.f;
          side->m[lane] = m_ref;
          side->l[lane] = l;
          fence_proxy_async_smem();           // generic writes -> visible to the bulk copies
          __syncwarp();
          if (lane == 0 && !*abort_flag) {
            const uint32_t dst = p_remote + (uint32_t)(hs * Cfg::PSLOT);
            const uint32_t bar = pf_remote + (uint32_t)(hs * 8);
            bulk_copy_to_cta(dst + q * 4096, stg, 4096, bar);
            bulk_copy_to_cta(dst + Cfg::PH + q * 512, side, 512, bar);
            bulk_commit_group();
            copies = true;
          }
        }
        ++segi;
      }
      if (lane == 0 && copies) bulk_wait_all();   // every copy into the peer has landed
      __syncwarp();
    }
  } else {
    // =========================================================================================
    // value CTA
    // =========================================================================================
    const uint32_t tO = tmem;   // all 512 columns
    uint8_t* sP = smem + Cfg::V_OFF_P;
    uint8_t* sV = smem + Cfg::V_OFF_V;
    if (warp == 0 && lane == 0) {
      // ------------------------------- TMA producer -------------------------------
      // per half tile (64 positions): two units of 256 latent columns, each four 64-column boxes
      DecWalk w;
      w.begin(p, u0, u1);
      DecSeg sg;
      int64_t n = 0;
      bool ok = true;
      while (ok && w.next(p, sg)) {
        for (int tt = 0; tt < sg.ntl && ok; ++tt) {
          for (int hh = 0; hh < 2 && ok; ++hh) {
            const int y = (int)(sg.sstart + (int64_t)(sg.tile0 + tt) * DEC_BT + hh * DEC_HT);
            for (int nh = 0; nh < 2; ++nh, ++n) {
              const int s = (int)(n % NV);
              if (n >= NV && !wait_bar(&bars->v_empty[s], (uint32_t)((n / NV) - 1) & 1u)) { ok = false; break; }
              mbar_arrive_expect_tx(&bars->v_full[s], Cfg::UNIT);
              uint8_t* dst = sV + s * Cfg::UNIT;
#pragma unroll
              for (int bx = 0; bx < 4; ++bx)
                tma_load_2d(dst + bx * (DEC_HT * 128), &tv, &bars->v_full[s], nh * 256 + bx * 64, y);
            }
          }
        }
      }
      if (*abort_flag) {
        for (int64_t i = (n > NV ? n - NV : 0); i < n; ++i)
          (void)mbar_wait(&bars->v_full[i % NV], (uint32_t)(i / NV) & 1u, drain_ns, p.status);
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------- P.C issuer -------------------------------
      // O[:, 256 nh + ...] += P (128 x 64, K-major, from the P slot) . C (64 x 256, MN-major, the unit)
      constexpr uint32_t idesc = idesc_bf16_f32(128, 256, false, true);
      const uint64_t pd0 = smem_desc_sw128(smem_u32(sP), 16, 1024);
      const uint64_t vd0 = smem_desc_sw128(smem_u32(sV), DEC_HT * 128, 1024);
      DecWalk w;
      w.begin(p, u0, u1);
      DecSeg sg;
      int64_t n = 0, i = 0;
      int segi = 0, fixes = 0;
      bool ok = true;
      while (ok && w.next(p, sg)) {
        for (int tt = 0; tt < sg.ntl && ok; ++tt) {
          for (int hh = 0; hh < 2; ++hh, ++i) {
            const int hs = (int)(i % NPH);
            if (!wait_bar(&bars->p_full[hs], (uint32_t)(i / NPH) & 1u)) { ok = false; break; }
            const bool first = tt == 0 && hh == 0;
            // the previous segment's epilogue must have read O before this segment overwrites it
            if (first && segi > 0 && !wait_bar(&bars->o_free, (uint32_t)(segi - 1) & 1u)) { ok = false; break; }
            const DecSide* sd = reinterpret_cast<const DecSide*>(sP + hs * Cfg::PSLOT + Cfg::PH);
            const int any = sd[0].flag | sd[1].flag | sd[2].flag | sd[3].flag;
            if (any) {
              // rows move their reference maximum here: O (every P.C so far) is rescaled first
              mma_commit(&bars->o_fix);
              if (!wait_bar(&bars->fix_done, (uint32_t)fixes & 1u)) { ok = false; break; }
              ++fixes;
            }
            tc_fence_after();
            const uint64_t pd = pd0 + (uint64_t)((hs * Cfg::PSLOT) >> 4);
            for (int nh = 0; nh < 2; ++nh, ++n) {
              const int s = (int)(n % NV);
              if (!wait_bar(&bars->v_full[s], (uint32_t)(n / NV) & 1u)) { ok = false; break; }
              tc_fence_after();
              const uint64_t vd = vd0 + (uint64_t)((s * Cfg::UNIT) >> 4);
#pragma unroll
              for (int kk = 0; kk < DEC_HT / 16; ++kk)
                mma_bf16_ss(tO + nh * 256, pd + (uint64_t)(kk * 2), vd + (uint64_t)(kk * (2048 >> 4)), idesc,
                            (first && kk == 0) ? 0u : 1u);
              mma_commit(&bars->v_empty[s]);
            }
            if (!ok) break;
            mma_commit(&bars->pfree[hs]);
            if (tt + 1 == sg.ntl && hh == 1) mma_commit(&bars->o_fin);
          }
        }
        ++segi;
      }
      if (!ok || *abort_flag) {
        *abort_flag = 1;
        mma_commit(&bars->drain[1]);
        (void)mbar_wait(&bars->drain[1], 0, drain_ns, p.status);
      }
    } else if (warp == 2 && lane == 0) {
      // ------------------------------- slot hand-back -------------------------------
      // once P.C has read a P slot and the rescale / epilogue warps have read its side data: re-arm
      // the slot's landing barrier for its next use, then tell the score CTA it may write the slot
      const uint32_t pe_remote = map_to_cta(smem_u32(&bars->p_empty[0]), 0);
      DecWalk w;
      w.begin(p, u0, u1);
      DecSeg sg;
      int64_t total = 0;
      while (w.next(p, sg)) total += 2 * (int64_t)sg.ntl;
      for (int64_t i = 0; i < total; ++i) {
        const int hs = (int)(i % NPH);
        if (!wait_bar(&bars->pfree[hs], (uint32_t)(i / NPH) & 1u)) break;
        if (i + NPH < total) {
          mbar_arrive_expect_tx(&bars->p_full[hs], Cfg::PSLOT);
          mbar_arrive_remote_release(pe_remote + (uint32_t)(hs * 8));
        }
      }
    } else if (warp >= 4) {
      // ------------------------------- rescale and epilogue -------------------------------
      const int w8 = warp - 4, q = w8 & 3, hc = w8 >> 2;
      const int row = q * 32 + lane;
      const uint32_t lane_off = (uint32_t)(q * 32) << 16;
      const uint32_t tcol = tO + lane_off + hc * 256;
      DecWalk w;
      w.begin(p, u0, u1);
      DecSeg sg;
      int64_t i = 0;
      int segi = 0, fixes = 0;
      while (w.next(p, sg)) {
        for (int tt = 0; tt < sg.ntl; ++tt) {
          for (int hh = 0; hh < 2; ++hh, ++i) {
            const int hs = (int)(i % NPH);
            (void)wait_bar(&bars->p_full[hs], (uint32_t)(i / NPH) & 1u);
            uint8_t* slot = sP + hs * Cfg::PSLOT;
            const DecSide* sd = reinterpret_cast<const DecSide*>(slot + Cfg::PH);
            const int any = sd[0].flag | sd[1].flag | sd[2].flag | sd[3].flag;
            if (any) {
              const bool ok = wait_bar(&bars->o_fix, (uint32_t)fixes & 1u);
              ++fixes;
              tc_fence_after();
              if (ok && sd[q].flag) {
                const float alpha = sd[q].alpha[lane];
#pragma unroll 1
                for (int cc = 0; cc < 256; cc += 32) {
                  uint32_t r[32];
                  tmem_ld32(tcol + cc, r);
                  tmem_wait_ld();
#pragma unroll
                  for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
                  tmem_st32(tcol + cc, r);
                }
                tmem_wait_st();
              }
              tc_fence_before();
              __syncwarp();
              if (lane == 0 && !*abort_flag) mbar_arrive(&bars->fix_done);
            }
            if (tt + 1 == sg.ntl && hh == 1) {
              // ---- epilogue of the segment: O / l (whole block) or the partial (O, m, l)
              const float m_ref = sd[q].m[lane];
              const float ltot = sd[q].l[lane];
              const bool ok = wait_bar(&bars->o_fin, (uint32_t)segi & 1u);
              tc_fence_after();
              const int ri = sg.rb * DEC_ROWS + row;
              const int rows_seq = p.n_q * p.H;
              const int64_t orow = (int64_t)sg.b * rows_seq + ri;
              const int slotp = 2 * pair + (segi == 0 ? 0 : 1);
              const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
              const float mul = sg.complete ? inv : 1.f;
              // this slot stays with this CTA until the epilogue is done: each warp turns its rows
              // around in 2 KB of it (32 rows x 16 columns, fp32) for stores of 64 B per row
              uint8_t* wst = slot + w8 * 2048;
#pragma unroll 1
              for (int cc = 0; cc < 256; cc += 16) {
                uint32_t r[16];
                tmem_ld16(tcol + cc, r);
                tmem_wait_ld();
                if (ok) {
#pragma unroll
                  for (int c = 0; c < 4; ++c)
                    *reinterpret_cast<float4*>(wst + lane * 64 + ((c ^ ((lane >> 1) & 3)) * 16)) =
                        make_float4(__uint_as_float(r[4 * c]) * mul, __uint_as_float(r[4 * c + 1]) * mul,
                                    __uint_as_float(r[4 * c + 2]) * mul, __uint_as_float(r[4 * c + 3]) * mul);
                }
                __syncwarp();
                if (ok) {
#pragma unroll
                  for (int j = 0; j < 4; ++j) {
                    const int rr = 8 * j + (lane >> 2);       // row within the warp's 32
                    const int c = lane & 3;
                    const float4 v = *reinterpret_cast<const float4*>(wst + rr * 64 + ((c ^ ((rr >> 1) & 3)) * 16));
                    const int rw = q * 32 + rr;               // row within the block
                    float* d;
                    bool write;
                    if (sg.complete) {
                      write = sg.rb * DEC_ROWS + rw < rows_seq;
                      d = p.out_lat + ((int64_t)sg.b * rows_seq + sg.rb * DEC_ROWS + rw) * DEC_DC;
                    } else {
                      write = true;
                      d = p.o_part + ((int64_t)slotp * DEC_ROWS + rw) * DEC_DC;
                    }
                    if (write) *reinterpret_cast<float4*>(d + hc * 256 + cc + 4 * c) = v;
                  }
                }
                __syncwarp();
              }
              if (ok && hc == 0) {
                if (sg.complete) {
                  if (ri < rows_seq && p.lse)
                    p.lse[orow] = ltot > 0.f ? (m_ref + log2f(ltot)) * 0.69314718055994531f : -INFINITY;
                } else {
                  p.m_part[(int64_t)slotp * DEC_ROWS + row] = m_ref;
                  p.l_part[(int64_t)slotp * DEC_ROWS + row] = ltot;
                }
              }
              fence_proxy_async_smem();     // the slot's generic accesses come before the next copies into it
              tc_fence_before();
              __syncwarp();
              if (lane == 0 && !*abort_flag) mbar_arrive(&bars->o_free);
            }
            __syncwarp();
            if (lane == 0 && !*abort_flag) mbar_arrive(&bars->pfree[hs]);
          }
        }
        ++segi;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();     // the score CTA's copies into the value CTA have landed (each issuer waited)
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------------------
// combine: 16 CTAs per block (8 rows each); merges the partials of blocks split across clusters and writes
// zeros / -inf for blocks with nothing to attend to
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) decode_combine_tc_kernel(DecParams p) {
  __shared__ int slots[256];
  __shared__ float wts[8][256];
  __shared__ int nsl;
  griddep_wait();
  griddep_launch_dependents();
  const int k = blockIdx.x;
  const int r0 = blockIdx.y * 8;     // this CTA's 8 rows of the block (one per warp)
  const int64_t bstart = p.prefix[k], bend = p.prefix[k + 1];
  const int b = k / p.nbps, rb = k % p.nbps;
  const int rows_seq = p.n_q * p.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (bend == bstart) {
    for (int r = r0 + warp; r < r0 + 8; r += 8) {
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
  if (threadIdx.x == 0) {
    // the partial of cluster q for this block: its first segment (slot 2q) unless the block
    // started inside q's range (then it is q's last segment, slot 2q + 1); clusters without work
    // are skipped
    int n = 0;
    for (int q = p0; q <= p1 && n < 256; ++q) {
      const int64_t qs = range_start(U, p.G, q);
      if (range_start(U, p.G, q + 1) == qs) continue;
      slots[n++] = (q == p0 && bstart > qs) ? 2 * q + 1 : 2 * q;
    }
    nsl = n;
  }
  __syncthreads();
  const int n = nsl;
  for (int r = r0 + warp; r < r0 + 8; r += 8) {
    const int ri = rb * DEC_ROWS + r;
    if (ri >= rows_seq) break;
    float M = -INFINITY;
    for (int i = lane; i < n; i += 32) M = fmaxf(M, p.m_part[(int64_t)slots[i] * DEC_ROWS + r]);
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float L = 0.f;
    for (int i = lane; i < n; i += 32) {
      const float m = p.m_part[(int64_t)slots[i] * DEC_ROWS + r];
      const float w = m == -INFINITY ? 0.f : ex2(m - M);
      wts[warp][i] = w;
      L += w * p.l_part[(int64_t)slots[i] * DEC_ROWS + r];
    }
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    __syncwarp();
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const int64_t orow = (int64_t)b * rows_seq + ri;
    float4* dst = reinterpret_cast<float4*>(p.out_lat + orow * DEC_DC);
    for (int d4 = lane; d4 < DEC_DC / 4; d4 += 32) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int i = 0; i < n; ++i) {
        const float w = wts[warp][i];
        if (w == 0.f) continue;
        const float4 o = reinterpret_cast<const float4*>(p.o_part + ((int64_t)slots[i] * DEC_ROWS + r) * DEC_DC)[d4];
        acc.x += w * o.x; acc.y += w * o.y; acc.z += w * o.z; acc.w += w * o.w;
      }
      dst[d4] = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
    if (lane == 0 && p.lse) p.lse[orow] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------------------------
static int g_decode_clusters_override = 0;

void set_decode_clusters(int n) { g_decode_clusters_override = n > 0 ? (n > 256 ? 256 : n) : 0; }

bool tc_decode_supported(const DecodeArgs& a) {
  if (!(a.dc == DEC_DC && (a.dr == 0 || a.dr == 64) && a.H > 0 && a.n_q > 0 && a.total_rows > 0 &&
        (int64_t)a.batch * a.n_q * a.H < (1LL << 31) - DEC_ROWS && a.total_rows < (1LL << 31) - DEC_BT))
    return false;
  // the plan stores tile prefixes in int32: the units of all blocks must stay below 2^31
  const int64_t nblocks = (int64_t)a.batch * ceil_div((int64_t)a.n_q * a.H, DEC_ROWS);
  const int64_t tiles = std::max<int64_t>(1, ceil_div(a.max_seqlen, DEC_BT));
  return nblocks < (1LL << 31) / tiles;
}

struct TcDecodePlan {
  int nbps, nblocks, G;
  size_t off_prefix, off_o, off_m, off_l, total;
};

template <int DR>
static int max_active_clusters_t() {
  int n = 0;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
  cfg.blockDim = dim3(DEC_THREADS, 1, 1);
  cfg.dynamicSmemBytes = DecCfg<DR>::SMEM;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaFuncSetAttribute(tc_decode_kernel<DR>, cudaFuncAttributeMaxDynamicSharedMemorySize, DecCfg<DR>::SMEM);
  const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, (void*)tc_decode_kernel<DR>, &cfg);
  if (e != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = sm_count() / 2;
  }
  return n;
}

// clusters of two CTAs that can be resident at once (the kernel is persistent: more would run as a
// second wave); computed once per device and tile variant
static int max_active_clusters(int dr) {
  static int cached[64][2] = {{0}};
  const int dev = current_device();
  const int v = dr == 0 ? 0 : 1;
  if (dev < 0 || dev >= 64) return sm_count() / 2;
  if (cached[dev][v] == 0) cached[dev][v] = dr == 0 ? max_active_clusters_t<0>() : max_active_clusters_t<64>();
  return cached[dev][v];
}

static TcDecodePlan plan_tc(const DecodeArgs& a) {
  TcDecodePlan t;
  t.nbps = (int)ceil_div((int64_t)a.n_q * a.H, DEC_ROWS);
  t.nblocks = a.batch * t.nbps;
  const int64_t units_max = (int64_t)t.nblocks * std::max<int64_t>(1, ceil_div(a.max_seqlen, DEC_BT));
  const int maxc = max_active_clusters(a.dr);
  int G = maxc;
  // Equal-length sequences with one row block each: give every block the same number of clusters
  // (no block is split unevenly and, with one cluster per block, no partials are written at all).
  const bool equal_blocks = a.total_rows == (int64_t)a.batch * a.max_seqlen && (!a.causal || t.nbps == 1);
  if (equal_blocks && t.nblocks <= maxc) G = t.nblocks * (maxc / t.nblocks);
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
static int launch_decode_t(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tqr,
                           const DecParams& p, cudaStream_t s) {
  static bool attr_set[64] = {false};
  const int dev = current_device();
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(tc_decode_kernel<DR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DecCfg<DR>::SMEM) != cudaSuccess)
      return MLA_ERR_CUDA;
    attr_set[dev] = true;
  }
  return launch_pdl(tc_decode_kernel<DR>, dim3(2 * p.G), dim3(DEC_THREADS), (size_t)DecCfg<DR>::SMEM, s, tk, tv,
                    tqr, p);
}

int tc_decode_launch(const DecodeArgs& a, cudaStream_t s) {
  const TcDecodePlan t = plan_tc(a);
  const int W = a.dc + a.dr;
  char* ws = static_cast<char*>(a.workspace);
  DecParams p{};
  p.q_abs = static_cast<const __nv_bfloat16*>(a.q_abs);
  p.q_rows = (int64_t)a.batch * a.n_q * a.H;
  p.W = W;
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

  // the cache: 128-position boxes of 64 columns for the score CTA, 64-position boxes for the value CTA;
  // the rotary query: 128 rows x 64 columns. All 128-byte swizzled (the MMA operand layout).
  CUtensorMap tk, tv, tqr;
  const uint64_t rows = (uint64_t)std::max<int64_t>(a.total_rows, 1);
  {
    const uint64_t dims[2] = {(uint64_t)W, rows};
    const uint64_t st[1] = {(uint64_t)W * 2};
    const uint32_t box[2] = {64, DEC_BT};
    if (!encode_tmap_bf16(&tk, const_cast<void*>(a.cache), 2, dims, st, box)) return MLA_ERR_CUDA;
  }
  {
    const uint64_t dims[2] = {(uint64_t)W, rows};
    const uint64_t st[1] = {(uint64_t)W * 2};
    const uint32_t box[2] = {64, DEC_HT};
    if (!encode_tmap_bf16(&tv, const_cast<void*>(a.cache), 2, dims, st, box)) return MLA_ERR_CUDA;
  }
  tqr = tk;
  if (a.dr) {
    const uint64_t dims[2] = {(uint64_t)W, (uint64_t)a.batch * a.n_q * a.H};
    const uint64_t st[1] = {(uint64_t)W * 2};
    const uint32_t box[2] = {64, DEC_ROWS};
    if (!encode_tmap_bf16(&tqr, const_cast<void*>(a.q_abs), 2, dims, st, box)) return MLA_ERR_CUDA;
  }
  int st0 = launch_pdl(decode_plan_kernel, dim3(1), dim3(1024), 0, s, p, const_cast<int32_t*>(p.prefix));
  if (st0) return st0;
  int st = a.dr == 0 ? launch_decode_t<0>(tk, tv, tqr, p, s) : launch_decode_t<64>(tk, tv, tqr, p, s);
  if (st) return st;
  // 16 CTAs per block (8 rows each): a split block's merge reads 2-3 partial slots of 256 KB
  return launch_pdl(decode_combine_tc_kernel, dim3((unsigned)t.nblocks, DEC_ROWS / 8), dim3(256), 0, s, p);
}

}  // namespace mla
