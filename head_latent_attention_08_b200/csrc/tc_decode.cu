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
//  * TMEM (512 columns) cannot hold O (128 x 512 fp32) next to S, so a CLUSTER OF TWO CTAs shares a
//    block: CTA r owns latent columns [256 r, 256 r + 256) and rotary columns [512 + 32 r, +32). Each
//    streams only its own columns of every cache tile (each cache byte crosses HBM once), computes the
//    partial S over them, and the two partials (rounded to fp16) are exchanged through distributed
//    shared memory; both CTAs form the same S = fp16(S0) + fp16(S1), run the same fp32 online
//    softmax and accumulate their half of O = P . C in TMEM (256 columns).
//  * The first 128 of this CTA's 256 latent query columns live in TMEM (64 columns of packed bf16,
//    the A operand of QK^T straight from TMEM), the other 128 and the rotary columns in shared memory
//    (brought by TMA). P (bf16) is written over its S tile and is the A operand of P . C from TMEM.
//    TMEM: Q 64 + O 256 + three 64-column S/P slots = 512 columns, so three tiles are between QK^T
//    and P.C at once. Shared memory: the query half, four cache stages and one receive and one
//    send-staging slot for the fp16 scores.
//  * O is rescaled only when a row's running maximum grows by more than 2^8 (the result is exact:
//    numerator and denominator share the stale reference maximum).
//  * Work: the (block, 64-position tile) units of all sequences are split evenly over the clusters
//    (persistent). A cluster that covers a whole block writes the normalised result; split blocks
//    leave (O, max, sum) partials that a combine kernel merges.
//  * Warp roles per CTA (512 threads): warp 0 lane 0 issues TMA loads, warp 1 lane 0 every QK^T and
//    warp 2 lane 0 every P.C, warps 12-15 send the partial scores (rounded to fp16; each warp copies
//    its 32 rows to the peer with one bulk copy and never waits on the peer), warps 4-11 form two
//    softmax warpgroups (thread = row = TMEM lane): warpgroup wg loads its 64 of the query's TMEM
//    columns at each segment, adds its own and the peer's fp16 partials of score columns
//    [32 wg, 32 wg + 32), meets the other warpgroup once per tile for the row maximum, writes P and
//    runs the epilogue.
//  * Every wait is bounded (global-timer limit); a wait that gives up sets the library's status word,
//    and the CTA abandons its work, drains its own TMA loads and MMAs and exits through the cluster
//    barrier.
#include <math.h>

#include <algorithm>

#include "sm100.cuh"
#include "tc.cuh"

namespace mla {

using namespace sm100;

constexpr int DEC_BT = 64;          // positions per tile
constexpr int DEC_THREADS = 512;   // warp 0 TMA, warp 1 MMA, warps 4-11 softmax, warps 12-15 query + sender
constexpr int DEC_DC = 512;         // latent width handled by this kernel
constexpr int DEC_HALF = 256;       // latent columns per CTA
constexpr int DEC_ROWS = 128;       // rows per block
constexpr int DEC_PREFETCH = 4;     // tiles brought into L2 beyond the shared-memory ring
constexpr int DEC_SLOTS = 3;        // S/P slots in TMEM: tiles between QK^T and P.C at once
constexpr int DEC_XSLOTS = 1;       // score-exchange slots (receive + send staging) in shared memory

template <int DR>
struct DecCfg {
  static constexpr int QL_BOX = DEC_ROWS * 128;         // 128 rows x 64 latent query columns (128 B)
  static constexpr int QR_BOX = DR ? 128 * 64 : 0;      // this CTA's 32 rotary query columns, 128 x 64 B
  static constexpr int K_BOX = DEC_BT * 128;            // 64 positions x 64 latent columns (128 B)
  static constexpr int KR_BOX = DR ? DEC_BT * 64 : 0;   // 64 positions x 32 rotary columns (64 B)
  static constexpr int STAGE_BYTES = 4 * K_BOX + KR_BOX;
  static constexpr int STAGES = 4;
  static constexpr int X_TILE = DEC_ROWS * DEC_BT * 2;   // one tile of partial scores, fp16, rows of 128 B
  static constexpr int OFF_QL = 0;                       // latent query columns [128, 256) of this CTA
  static constexpr int OFF_QR = 2 * QL_BOX;
  static constexpr int OFF_K = OFF_QR + QR_BOX;
  static constexpr int OFF_X = OFF_K + STAGES * STAGE_BYTES;
  static constexpr int OFF_XS = OFF_X + DEC_XSLOTS * X_TILE;   // receive slots, then send stagings
  static constexpr int OFF_BAR = OFF_XS + DEC_XSLOTS * X_TILE;
  static constexpr int OFF_RED = OFF_BAR + 256;          // row maxima [2][2][128], row sums [2][128]
  static constexpr int SMEM = OFF_RED + 6 * DEC_ROWS * 4 + 1024;
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
    tc_decode_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tkr,
                     const __grid_constant__ CUtensorMap tqr, const __grid_constant__ CUtensorMap tql,
                     DecParams p) {
  using Cfg = DecCfg<DR>;
  constexpr int ST = Cfg::STAGES;
  constexpr int NS = DEC_SLOTS;
  constexpr int XS = DEC_XSLOTS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQL = smem + Cfg::OFF_QL;
  uint8_t* sQR = smem + Cfg::OFF_QR;
  uint8_t* sK = smem + Cfg::OFF_K;
  uint8_t* sX = smem + Cfg::OFF_X;
  float* red = reinterpret_cast<float*>(smem + Cfg::OFF_RED);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* k_full = bars;              // [ST] cache tile landed
  uint64_t* k_empty = k_full + ST;      // [ST] cache tile consumed by its P.C
  uint64_t* qr_full = k_empty + ST;     // query columns in shared memory landed (TMA)
  uint64_t* ql_full = qr_full + 1;      // latent query columns written to TMEM (softmax warps)
  uint64_t* q_empty = ql_full + 1;      // last QK^T of a segment done: the query may be replaced
  uint64_t* s_full = q_empty + 1;       // [NS] partial S of a slot computed (MMA -> sender)
  uint64_t* own_ready = s_full + NS;    // [NS] own fp16 partials staged, S read (sender -> softmax)
  uint64_t* p_full = own_ready + NS;    // [NS] P written (softmax -> MMA)
  uint64_t* o_done = p_full + NS;       // [NS] the P.C of a tile of this slot completed
  uint64_t* x_full = o_done + NS;       // [XS] peer's partial scores arrived (transaction count)
  uint64_t* x_empty = x_full + XS;      // [XS] both softmaxes have read this CTA's scores
  uint64_t* drain = x_empty + XS;       // [2] MMA drain on abort, one per issuing thread
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int pair = blockIdx.x >> 1;
  const int dim0 = rank == 0 ? 0 : DEC_HALF;           // first latent column of this CTA
  const int rdim0 = DEC_DC + (int)rank * (DR / 2);     // first rotary column of this CTA

  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    mbar_init(qr_full, 1);
    mbar_init(ql_full, 8);            // one arrival per softmax warp (each writes its rows' half)
    mbar_init(q_empty, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&own_ready[s], 4);    // one arrival per sender warp
      mbar_init(&p_full[s], 8);       // one arrival per softmax warp
      mbar_init(&o_done[s], 1);
    }
    for (int s = 0; s < XS; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], 2);      // the peer's softmax (remote) and this CTA's (local)
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    // arm the first use of each receive slot: one local arrival plus the peer's four 4 KB bulk copies
    for (int s = 0; s < XS; ++s) mbar_arrive_expect_tx(&x_full[s], Cfg::X_TILE);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tk);
    prefetch_tmap(&tql);
    if (DR) {
      prefetch_tmap(&tkr);
      prefetch_tmap(&tqr);
    }
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();           // the peer's barriers are initialised before any remote access
  tc_fence_after();
  griddep_wait();           // the plan, the query block and the cache come from earlier kernels
  griddep_launch_dependents();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tQ = tmem;               // columns [0, 64): this CTA's latent query columns [0, 128), bf16 pairs
  const uint32_t tO = tmem + 64;          // columns [64, 320): this CTA's half of O
  const uint32_t tS = tmem + 320;         // columns [320, 512): three 64-column S / P slots

  const int64_t U = p.prefix[p.nblocks];
  const int64_t u0 = range_start(U, p.G, pair), u1 = range_start(U, p.G, pair + 1);
  const int64_t n_total = u1 - u0;
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
      {
        // the query columns that QK^T reads from shared memory: latent [128, 256) of this CTA and
        // its rotary columns, once the previous segment's last QK^T is done
        const int qrow = (int)((int64_t)b * p.n_q * p.H + (int64_t)rb * DEC_ROWS);
        if (seg > 0 && (*abort_flag || !mbar_wait(q_empty, (seg - 1) & 1, p.wait_ns, p.status))) { ok = false; break; }
        mbar_arrive_expect_tx(qr_full, 2 * Cfg::QL_BOX + Cfg::QR_BOX);
        for (int kb = 0; kb < 2; ++kb) tma_load_2d(sQL + kb * Cfg::QL_BOX, &tql, qr_full, dim0 + 128 + kb * 64, qrow);
        if (DR) tma_load_2d(sQR, &tqr, qr_full, rdim0, qrow);
        ++q_loads;
      }
      int pf_next = 0;                      // next tile of this segment to warm in L2
      for (int tt = 0; tt < ntl; ++tt, ++g) {
        const int s = (int)(g % ST);
        if (g >= ST && (*abort_flag || !mbar_wait(&k_empty[s], (int)((g / ST) - 1) & 1, p.wait_ns, p.status))) {
          ok = false;
          break;
        }
        // the first query block is read by the softmax warps at the same time: hold the rest of the
        // ring until it is in, so that it does not queue behind four tiles of every CTA
        if (g == 1 && (*abort_flag || !mbar_wait(ql_full, 0, p.wait_ns, p.status))) {
          ok = false;
          break;
        }
        if (g >= ST) {
          // warm L2 for up to DEC_PREFETCH tiles beyond the shared-memory ring, at most two per step:
          // while the ring first fills, nothing is prefetched, so that the first tiles of all CTAs do
          // not queue behind a burst of prefetches
          if (pf_next < tt + ST) pf_next = tt + ST;
          const int pf_end = min(ntl, tt + ST + DEC_PREFETCH);
          for (int n = 0; n < 2 && pf_next < pf_end; ++n, ++pf_next) {
            const int yp = (int)(sstart + (int64_t)(tile0 + pf_next) * DEC_BT);
            for (int kb = 0; kb < 4; ++kb) tma_prefetch_2d(&tk, dim0 + kb * 64, yp);
            if (DR) tma_prefetch_2d(&tkr, rdim0, yp);
          }
        }
        uint8_t* dst = sK + s * Cfg::STAGE_BYTES;
        mbar_arrive_expect_tx(&k_full[s], Cfg::STAGE_BYTES);
        const int y = (int)(sstart + (int64_t)(tile0 + tt) * DEC_BT);
        for (int kb = 0; kb < 4; ++kb) tma_load_2d(dst + kb * Cfg::K_BOX, &tk, &k_full[s], dim0 + kb * 64, y);
        if (DR) tma_load_2d(dst + 4 * Cfg::K_BOX, &tkr, &k_full[s], rdim0, y);
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
      if (q_loads > 0) (void)mbar_wait(qr_full, (q_loads - 1) & 1, drain_ns, p.status);
    }
  } else if ((warp == 1 || warp == 2) && lane == 0) {
    // ------------------------------- MMA issuers -------------------------------
    // Two threads issue the MMAs (one thread alone issues about one MMA per 50-90 cycles, and QK^T is
    // 18 MMAs): warp 1 issues QK^T of every tile, warp 2 P.C of every tile. Tile g's QK^T writes the
    // S/P slot that P.C of tile g - NS read, so it waits for that P.C to complete (its o_done phase).
    // P.C of tile g reads the cache stage that QK^T of tile g read as well; QK^T completed before the
    // softmax could write P (s_full), so the stage's release after P.C covers both readers. Only
    // warp 2 accumulates into O, in issue order.
    // Each thread's scalar work sits between consecutive MMAs: descriptors are built once for stage 0
    // and advanced by constant offsets (the 14-bit start-address field holds shared addresses >> 4
    // below 256 KB, so the additions never carry into the other fields).
    const bool qk_issuer = warp == 1;
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, DEC_BT, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, DEC_HALF, false, true);
    constexpr uint64_t kStage = (uint64_t)(Cfg::STAGE_BYTES >> 4);
    const uint32_t qr_base = smem_u32(sQR), k_base = smem_u32(sK);
    const uint64_t qld0 = smem_desc_sw128(smem_u32(sQL), 16, 1024);          // latent query [128, 256), K-major (A)
    const uint64_t kd0 = smem_desc_sw128(k_base, 16, 1024);                  // cache tile, K-major (B of QK^T)
    const uint64_t cd0 = smem_desc_sw128(k_base, Cfg::K_BOX, 1024);          // cache tile, MN-major (B of P.C)
    const uint64_t rd0 = smem_desc_sw64(k_base + 4 * Cfg::K_BOX, 16, 512);   // rotary columns of the tile
    const uint64_t qd0 = smem_desc_sw64(qr_base, 16, 512);                   // rotary query columns
    auto wait_mma = [&](uint64_t* bar, uint32_t parity) -> bool {
      return !*abort_flag && mbar_wait(bar, parity, p.wait_ns, p.status);
    };
    // segments in tile order: [seg_start, seg_end) is the segment holding tile g
    int64_t useg = u0, seg_start = 0, seg_end = 0;
    int kseg = u0 < u1 ? find_block(p.prefix, p.nblocks, u0) : 0;
    int segi = -1;
    auto advance_segment = [&](int64_t g) {
      if (g < seg_end) return false;
      const int64_t bend = p.prefix[kseg + 1];
      const int64_t send = u1 < bend ? u1 : bend;
      seg_start = g;
      seg_end = g + (send - useg);
      ++segi;
      useg = send;
      if (useg < u1) kseg = find_block(p.prefix, p.nblocks, useg);
      return true;
    };
    bool ok = true;
    if (qk_issuer) {
      for (int64_t g = 0; g < n_total; ++g) {
        if (advance_segment(g)) {
          // this segment's query: TMEM half (softmax warps) and shared-memory half (TMA)
          if (!wait_mma(ql_full, (uint32_t)segi & 1u) || !wait_mma(qr_full, (uint32_t)segi & 1u)) { ok = false; break; }
        }
        const int s = (int)(g % ST);
        const int sl = (int)(g % NS);
        if (!wait_mma(&k_full[s], (uint32_t)(g / ST) & 1u)) { ok = false; break; }
        if (g >= NS && !wait_mma(&o_done[sl], (uint32_t)((g / NS) - 1) & 1u)) { ok = false; break; }
        tc_fence_after();
        const uint32_t td = tS + sl * 64;
        const uint64_t kd = kd0 + (uint64_t)s * kStage;
        // latent columns [0, 128) of this CTA: the query from TMEM; [128, 256): from shared memory
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(td, tQ + kb * 32 + kk * 8, kd + (uint64_t)((kb * Cfg::K_BOX + kk * 32) >> 4), idesc_qk,
                        (kb | kk) ? 1u : 0u);
        }
#pragma unroll
        for (int kb = 2; kb < 4; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(td, qld0 + (uint64_t)(((kb - 2) * Cfg::QL_BOX + kk * 32) >> 4),
                        kd + (uint64_t)((kb * Cfg::K_BOX + kk * 32) >> 4), idesc_qk, 1u);
        }
        if (DR) {
          // this CTA's 32 rotary columns: rows of 64 B, 8-row groups 512 B apart
          const uint64_t rd = rd0 + (uint64_t)s * kStage;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) mma_bf16_ss(td, qd0 + (uint64_t)(kk * 2), rd + (uint64_t)(kk * 2), idesc_qk, 1u);
        }
        mma_commit(&s_full[sl]);
        if (g + 1 == seg_end) mma_commit(q_empty);
      }
    } else {
      for (int64_t g = 0; g < n_total; ++g) {
        const bool first = advance_segment(g);   // the first tile of a segment opens O (accumulate = 0)
        const int s = (int)(g % ST);
        const int sl = (int)(g % NS);
        if (!wait_mma(&p_full[sl], (uint32_t)(g / NS) & 1u)) { ok = false; break; }
        tc_fence_after();
        // B = this CTA's 256 latent columns of the tile: MN-major, 64-column boxes K_BOX apart
        const uint64_t cd = cd0 + (uint64_t)s * kStage;
        const uint32_t ta = tS + sl * 64;
#pragma unroll
        for (int kk = 0; kk < DEC_BT / 16; ++kk)
          mma_bf16_ts(tO, ta + kk * 8, cd + (uint64_t)(kk * (2048 >> 4)), idesc_pv, (first && kk == 0) ? 0u : 1u);
        // the stage of a segment's last tile is released by the softmax warps after the epilogue,
        // which turns O around in it
        if (g + 1 != seg_end) mma_commit(&k_empty[s]);
        mma_commit(&o_done[sl]);
      }
    }
    if (!ok || *abort_flag) {
      *abort_flag = 1;
      // every MMA this thread issued must finish before TMEM is released
      uint64_t* d = &drain[qk_issuer ? 0 : 1];
      mma_commit(d);
      (void)mbar_wait(d, 0, drain_ns, p.status);
    }
  } else if (warp >= 12) {
    // -------------------------------- score sender --------------------------------
    // Thread = row = TMEM lane, and each warp handles its 32 rows on its own. For each tile: load this
    // CTA's partial scores (64 columns), round them to fp16 into the staging slot (the softmax reads
    // its own partials there) and send the warp's 32 rows (4 KB, both warpgroups' halves) to the
    // same slot of the peer with one bulk copy. The sender never waits for the peer's scores, so the
    // peer receives tile g as soon as this CTA's QK^T of tile g is done.
    const int quarter = warp - 12;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t x_remote = map_to_cta(smem_u32(sX), peer);
    const uint32_t xf_remote = map_to_cta(smem_u32(x_full), peer);
    const uint32_t xrow = (uint32_t)(row * 128);          // 64 fp16 per row: 8 chunks of 16 B
    const uint32_t xwarp = (uint32_t)(quarter * 32 * 128);// this warp's 32 rows: 4 KB of each slot
    const int swz = row & 7;                              // chunk swizzle against bank conflicts
    uint8_t* staging = smem + Cfg::OFF_XS;
    auto wait_cta = [&](uint64_t* bar, int parity) {
      if (*abort_flag) return;
      if (!mbar_wait(bar, (uint32_t)parity, p.wait_ns, p.status)) *abort_flag = 1;
    };
    for (int64_t g = 0; g < n_total; ++g) {
      const int sl = (int)(g % NS);         // S slot
      const int xs = (int)(g % XS);         // exchange slot
      wait_cta(&s_full[sl], (int)(g / NS) & 1);
      tc_fence_after();
      uint32_t h[32];                       // fp16 pairs: [0, 16) for warpgroup 0, [16, 32) for 1
      {
        uint32_t r0[32], r1[32];
        tmem_ld32(tS + lane_off + sl * 64, r0);
        tmem_ld32(tS + lane_off + sl * 64 + 32, r1);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          __half2 v0 = __floats2half2_rn(__uint_as_float(r0[2 * c]), __uint_as_float(r0[2 * c + 1]));
          __half2 v1 = __floats2half2_rn(__uint_as_float(r1[2 * c]), __uint_as_float(r1[2 * c + 1]));
          h[c] = *reinterpret_cast<uint32_t*>(&v0);
          h[16 + c] = *reinterpret_cast<uint32_t*>(&v1);
        }
      }
      // staging slot xs and the peer's receive slot xs were last used by tile g - XS: both this CTA's
      // softmax and the peer's have read that tile once x_empty completes (2 arrivals)
      if (g >= XS) wait_cta(&x_empty[xs], (int)((g / XS) - 1) & 1);
      {
        uint8_t* stg = staging + xs * Cfg::X_TILE + xrow;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(stg + ((c ^ swz) * 16)) =
              make_uint4(h[4 * c], h[4 * c + 1], h[4 * c + 2], h[4 * c + 3]);
      }
      fence_proxy_async_smem();             // generic writes -> visible to the bulk copies
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (!*abort_flag) {
          const uint32_t off = (uint32_t)(xs * Cfg::X_TILE) + xwarp;
          bulk_copy_to_cta(x_remote + off, staging + off, 32 * 128, xf_remote + xs * 8);
        }
        mbar_arrive(&own_ready[sl]);        // this warp's partials staged and read: P may overwrite
      }
    }
  } else if (warp >= 4) {
    // ---------------------------- softmax and epilogue ----------------------------
    // Two warpgroups share every tile: warpgroup wg owns score columns [32 wg, 32 wg + 32) of each
    // row (thread = row = TMEM lane), packed P columns [16 wg, 16 wg + 16) and O columns
    // [128 wg, 128 wg + 128). S = fp16(own partial) + fp16(peer's partial), both read from shared
    // memory (the sender's staging slot and the peer's copy), identically in both CTAs. The
    // warpgroups meet once per tile on the row maximum.
    const int wg = (warp - 4) >> 2;
    const int quarter = (warp - 4) & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    float* mx = red;                                      // [2 tiles][2 warpgroups][128]
    float* lx = red + 4 * DEC_ROWS;                       // [2 warpgroups][128]
    const uint8_t* staging = smem + Cfg::OFF_XS;
    const uint32_t xe_remote = map_to_cta(smem_u32(x_empty), peer);
    const uint32_t xrow = (uint32_t)(row * 128);
    const int swz = row & 7;
    int64_t g = 0, pv_waited = 0;
    int seg = 0;
    int64_t u = u0;
    int k = u0 < u1 ? find_block(p.prefix, p.nblocks, u0) : 0;
    // A wait that gives up sets the abort flag; from then on every wait is skipped but the loop
    // structure is walked unchanged, so that all threads keep meeting the same named barriers and
    // warp-collective TMEM instructions (no thread is left waiting). No barrier with a transaction
    // count is re-armed and no slot is released to the peer after an abort.
    auto wait_cta = [&](uint64_t* bar, int parity) {
      if (*abort_flag) return;
      if (!mbar_wait(bar, (uint32_t)parity, p.wait_ns, p.status)) *abort_flag = 1;
    };
    // this warpgroup's 64 of the CTA's first 128 latent query columns of block kq, into TMEM (the other
    // 128 come to shared memory by TMA), once the previous segment's last QK^T has read the query.
    // Thread = row = TMEM lane, but a load with one row per thread touches 32 rows per instruction, so
    // the rows are loaded 4 x 128 B per instruction and turned around in shared memory, swizzled
    // (chunk ^ row % 8: both the stores and the row reads are free of bank conflicts):
    //  * the first query of the CTA in this warp's 4 KB of cache stage 1, which the producer fills
    //    only once this query is in (ql_full);
    //  * a later one in this warp's 2 KB of the send-staging slot, in two rounds of 16 rows, once the
    //    exchange of the previous segment's last tile is complete (x_empty: the peer has read the
    //    copy, so no bulk copy still reads the slot; the sender writes it again only after the next
    //    QK^T, which needs this query).
    auto load_query = [&](int kq, int segment, int64_t g_prev) {
      const int bq = kq / p.nbps, rbq = kq % p.nbps;
      const int64_t qr0 = (int64_t)bq * p.n_q * p.H + (int64_t)rbq * DEC_ROWS + quarter * 32;   // warp's first row
      const int col0 = dim0 + wg * 64;
      if (segment > 0) wait_cta(q_empty, (segment - 1) & 1);
      tc_fence_after();
      uint4 v[8];
      const int chunk = lane & 7;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t qr = qr0 + 4 * j + (lane >> 3);
        const uint4* src = reinterpret_cast<const uint4*>(p.q_abs + qr * p.W + col0) + chunk;
        v[j] = qr < p.q_rows ? *src : make_uint4(0u, 0u, 0u, 0u);
      }
      uint32_t r[32];
      if (segment == 0) {
        uint8_t* scr = sK + Cfg::STAGE_BYTES + (warp - 4) * 4096;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int rr = 4 * j + (lane >> 3);
          *reinterpret_cast<uint4*>(scr + rr * 128 + ((chunk ^ (rr & 7)) * 16)) = v[j];
        }
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(scr + lane * 128 + ((c ^ (lane & 7)) * 16));
          r[4 * c] = w.x; r[4 * c + 1] = w.y; r[4 * c + 2] = w.z; r[4 * c + 3] = w.w;
        }
        fence_proxy_async_smem();           // these generic accesses come before the stage's TMA fill
        __syncwarp();
      } else {
        wait_cta(&x_empty[g_prev % XS], (int)((g_prev / XS) & 1));
        uint8_t* scr = smem + Cfg::OFF_XS + (warp - 4) * 2048;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int j = 4 * h; j < 4 * h + 4; ++j) {
            const int rr = 4 * j + (lane >> 3) - 16 * h;
            *reinterpret_cast<uint4*>(scr + rr * 128 + ((chunk ^ (rr & 7)) * 16)) = v[j];
          }
          __syncwarp();
          if ((lane >> 4) == h) {
            const int rr = lane - 16 * h;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 w = *reinterpret_cast<const uint4*>(scr + rr * 128 + ((c ^ (rr & 7)) * 16));
              r[4 * c] = w.x; r[4 * c + 1] = w.y; r[4 * c + 2] = w.z; r[4 * c + 3] = w.w;
            }
          }
          __syncwarp();
        }
      }
      tmem_st32(tQ + lane_off + wg * 32, r);   // 32 TMEM columns = 64 bf16
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ql_full);
    };
    if (u0 < u1) load_query(k, 0, 0);
    while (u < u1) {
      const int64_t bstart = p.prefix[k], bend = p.prefix[k + 1];
      const int64_t send_u = u1 < bend ? u1 : bend;
      const int tile0 = (int)(u - bstart), ntl = (int)(send_u - u);
      const bool complete = (u == bstart) && (send_u == bend);
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
      float m_ref = -INFINITY, l = 0.f;     // reference maximum (log2 units), this group's sum
      for (int tt = 0; tt < ntl; ++tt, ++g) {
        const int sl = (int)(g % NS);         // the tile's S / P slot
        const int xi = (int)(g % XS);         // the tile's exchange slot (this warpgroup reads its half)
        float s[32];
        wait_cta(&own_ready[sl], (int)(g / NS) & 1);
        tc_fence_after();
        uint4 own[4];
        {
          const uint8_t* xo = staging + xi * Cfg::X_TILE + xrow;
#pragma unroll
          for (int c = 0; c < 4; ++c) own[c] = *reinterpret_cast<const uint4*>(xo + (((4 * wg + c) ^ swz) * 16));
        }
        wait_cta(&x_full[xi], (int)(g / XS) & 1);
        {
          const uint8_t* xr = sX + xi * Cfg::X_TILE + xrow;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(xr + (((4 * wg + c) ^ swz) * 16));
            const uint32_t pv[4] = {v.x, v.y, v.z, v.w};
            const uint32_t ov[4] = {own[c].x, own[c].y, own[c].z, own[c].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              // the sum of the two fp16 partials, in fp16 (commutative: the same in both CTAs), then
              // widened once
              const __half2 sh = __hadd2(*reinterpret_cast<const __half2*>(&ov[j]),
                                         *reinterpret_cast<const __half2*>(&pv[j]));
              const float2 f = __half22float2(sh);
              s[8 * c + 2 * j] = f.x;
              s[8 * c + 2 * j + 1] = f.y;
            }
          }
        }
        // mask (only where the tile crosses a row's limit) and the raw row maximum
        const int t0 = (tile0 + tt) * DEC_BT + wg * 32;
        if (t0 + 32 > cnt) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (t0 + c >= cnt) s[c] = -INFINITY;
        }
        float m4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
        for (int c = 4; c < 32; c += 4) {
          m4[0] = fmaxf(m4[0], s[c]);
          m4[1] = fmaxf(m4[1], s[c + 1]);
          m4[2] = fmaxf(m4[2], s[c + 2]);
          m4[3] = fmaxf(m4[3], s[c + 3]);
        }
        float* mxs = mx + (g & 1) * 2 * DEC_ROWS;
        mxs[wg * DEC_ROWS + row] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        named_bar_sync(3, 256);               // both maxima are in; the slots of this tile are read
        if (wg == 0 && row == 0 && !*abort_flag) {
          // both warpgroups have read both slots (the barrier above); this thread's own wait saw the
          // receive slot's phase complete (the flag is still clear), so the re-arm cannot meet a phase
          // with bytes outstanding. Then release the slot to the peer's sender and the staging slot to
          // this CTA's sender.
          mbar_arrive_expect_tx(&x_full[xi], Cfg::X_TILE);
          mbar_arrive_remote(xe_remote + xi * 8);
          mbar_arrive(&x_empty[xi]);
        }
        const float mx_raw = fmaxf(mxs[row], mxs[DEC_ROWS + row]);
        const float mx_t = mx_raw * p.scale_log2;   // the scale is positive: the order is kept
        bool need = false;
        float factor = 1.f;
        if (mx_t > m_ref + 8.f) {
          if (m_ref != -INFINITY) {
            need = true;
            factor = ex2(m_ref - mx_t);
            l *= factor;
          }
          m_ref = mx_t;
        }
        const float mu = m_ref == -INFINITY ? 0.f : m_ref;
        // P in bf16 by truncation (the top half of each fp32: one byte permute per pair instead of a
        // conversion), and the row sum of the same truncated values, so that numerator and
        // denominator of the normalisation share the rounding
        float sum0 = 0.f, sum1 = 0.f;
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint32_t b0 = __float_as_uint(ex2(fmaf(s[2 * c], p.scale_log2, -mu))) & 0xFFFF0000u;
          const uint32_t b1 = __float_as_uint(ex2(fmaf(s[2 * c + 1], p.scale_log2, -mu))) & 0xFFFF0000u;
          sum0 += __uint_as_float(b0);
          sum1 += __uint_as_float(b1);
          pk[c] = __byte_perm(b0, b1, 0x7632);
        }
        l += sum0 + sum1;
        // P overwrites the S slot: the sender has read it (own_ready)
        tmem_st16(tS + lane_off + sl * 64 + wg * 16, pk);
        tmem_wait_st();
        // O may be touched only once every earlier P.C is done: needed when a row of this warp rescales,
        // and at the last tile of a segment. P.C of tile g - 1 commits to its slot's o_done barrier, whose
        // previous phase (P.C of tile g - 1 - NS) completed before QK^T of tile g - 1 could use the slot;
        // its completion implies every earlier P.C's (one issuing thread, in-order pipe).
        const bool rescale = __any_sync(0xffffffffu, need);
        if ((rescale || tt + 1 == ntl) && g > pv_waited) {
          wait_cta(&o_done[(g - 1) % NS], (int)(((g - 1) / NS) & 1));
          pv_waited = g;
        }
        tc_fence_after();
        if (rescale) {
#pragma unroll 1
          for (int cc = 0; cc < DEC_HALF / 2; cc += 32) {
            uint32_t r[32];
            tmem_ld32(tO + lane_off + wg * 128 + cc, r);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * factor);
            tmem_st32(tO + lane_off + wg * 128 + cc, r);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[sl]);   // this warp's rows of P are in (and O rescaled)
      }
      // the next segment's query can go in now (its QK^T overlaps this epilogue)
      const int k_next = send_u < u1 ? find_block(p.prefix, p.nblocks, send_u) : k;
      if (send_u < u1) load_query(k_next, seg + 1, g - 1);
      // epilogue of the segment: wait for its last P.C, then read this group's quarter of O
      if (g > pv_waited) {
        wait_cta(&o_done[(g - 1) % NS], (int)(((g - 1) / NS) & 1));
        pv_waited = g;
      }
      tc_fence_after();
      lx[wg * DEC_ROWS + row] = l;
      named_bar_sync(3, 256);
      const float ltot = lx[row] + lx[DEC_ROWS + row];
      const int64_t orow = (int64_t)b * p.n_q * p.H + ri;
      const int slot = 2 * pair + (seg == 0 ? 0 : 1);
      const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
      float* dst = complete ? p.out_lat + orow * DEC_DC + dim0 + wg * 128
                            : p.o_part + ((int64_t)slot * DEC_ROWS + row) * DEC_DC + dim0 + wg * 128;
      const float mul = complete ? inv : 1.f;
      const bool write = complete ? valid : true;
      const int s_last = (int)((g - 1) % ST);   // cache stage of the segment's last tile, held for us
      if (!*abort_flag) {
        // The segment's last P.C is done (above), and the P.C issuer left that tile's cache stage to
        // this epilogue. Each warp turns its 32 rows x 32 columns of O around in its 4 KB of the stage
        // (swizzled as for the query) and stores 4 rows x 128 B per instruction.
        uint8_t* wscratch = sK + s_last * Cfg::STAGE_BYTES + (warp - 4) * 4096;
        const int chunk = lane & 7;
#pragma unroll 1
        for (int cc = 0; cc < DEC_HALF / 2; cc += 32) {
          uint32_t r[32];
          tmem_ld32(tO + lane_off + wg * 128 + cc, r);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<float4*>(wscratch + lane * 128 + ((c ^ (lane & 7)) * 16)) =
                make_float4(__uint_as_float(r[4 * c]) * mul, __uint_as_float(r[4 * c + 1]) * mul,
                            __uint_as_float(r[4 * c + 2]) * mul, __uint_as_float(r[4 * c + 3]) * mul);
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int rr = 4 * j + (lane >> 3);            // row within the warp's 32
            const int rw = quarter * 32 + rr;              // row within the block
            const float4 w = *reinterpret_cast<const float4*>(wscratch + rr * 128 + ((chunk ^ (rr & 7)) * 16));
            float* d;
            bool ok_row;
            if (complete) {
              ok_row = rb * DEC_ROWS + rw < p.n_q * p.H;
              d = p.out_lat + ((int64_t)b * p.n_q * p.H + rb * DEC_ROWS + rw) * DEC_DC;
            } else {
              ok_row = true;
              d = p.o_part + ((int64_t)slot * DEC_ROWS + rw) * DEC_DC;
            }
            if (ok_row) *reinterpret_cast<float4*>(d + dim0 + wg * 128 + cc + chunk * 4) = w;
          }
          __syncwarp();
        }
      } else {
#pragma unroll 1
        for (int cc = 0; cc < DEC_HALF / 2; cc += 32) {
          uint32_t r[32];
          tmem_ld32(tO + lane_off + wg * 128 + cc, r);
          tmem_wait_ld();
          if (write) {
            float4* d4 = reinterpret_cast<float4*>(dst + cc);
#pragma unroll
            for (int c = 0; c < 8; ++c)
              d4[c] = make_float4(__uint_as_float(r[4 * c]) * mul, __uint_as_float(r[4 * c + 1]) * mul,
                                  __uint_as_float(r[4 * c + 2]) * mul, __uint_as_float(r[4 * c + 3]) * mul);
          }
        }
      }
      // hand the stage back to the producer: the generic accesses above come before its TMA fill
      fence_proxy_async_smem();
      named_bar_sync(3, 256);
      if (wg == 0 && row == 0) mbar_arrive(&k_empty[s_last]);
      if (rank == 0 && wg == 0) {
        if (complete) {
          if (valid && p.lse) p.lse[orow] = ltot > 0.f ? (m_ref + log2f(ltot)) * 0.69314718055994531f : -INFINITY;
        } else {
          p.m_part[(int64_t)slot * DEC_ROWS + row] = m_ref;
          p.l_part[(int64_t)slot * DEC_ROWS + row] = ltot;
        }
      }
      tc_fence_before();
      u = send_u;
      ++seg;
      k = k_next;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) {
    // abandoned work: let any bulk copy already issued between the pair land before either CTA
    // leaves (in normal operation every copy has been consumed before this point)
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 1000000ull) {
    }
  }
  __syncthreads();
  cluster_sync();     // the peer may write into this CTA's exchange buffer until it is done
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
  return a.dc == DEC_DC && (a.dr == 0 || a.dr == 64) && a.H > 0 && a.n_q > 0 && a.total_rows > 0 &&
         (int64_t)a.batch * a.n_q * a.H < (1LL << 31) - DEC_ROWS && a.total_rows < (1LL << 31) - DEC_BT;
}

struct TcDecodePlan {
  int nbps, nblocks, G;
  size_t off_prefix, off_o, off_m, off_l, total;
};

// clusters of two CTAs that can be resident at once (the kernel is persistent: more would run as a
// second wave); computed once per device and tile variant
static int max_active_clusters(int dr) {
  static int cached[64][2] = {{0}};
  const int dev = current_device();
  const int v = dr == 0 ? 0 : 1;
  if (dev < 0 || dev >= 64) return sm_count() / 2;
  if (cached[dev][v] == 0) {
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
    cfg.blockDim = dim3(DEC_THREADS, 1, 1);
    cfg.dynamicSmemBytes = dr == 0 ? DecCfg<0>::SMEM : DecCfg<64>::SMEM;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (dr == 0) {
      cudaFuncSetAttribute(tc_decode_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, DecCfg<0>::SMEM);
      e = cudaOccupancyMaxActiveClusters(&n, (void*)tc_decode_kernel<0>, &cfg);
    } else {
      cudaFuncSetAttribute(tc_decode_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, DecCfg<64>::SMEM);
      e = cudaOccupancyMaxActiveClusters(&n, (void*)tc_decode_kernel<64>, &cfg);
    }
    if (e != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = sm_count() / 2;
    }
    cached[dev][v] = n;
  }
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
static int launch_decode_t(const CUtensorMap& tk, const CUtensorMap& tkr, const CUtensorMap& tqr,
                           const CUtensorMap& tql, const DecParams& p, cudaStream_t s) {
  static bool attr_set[64] = {false};
  const int dev = current_device();
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(tc_decode_kernel<DR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DecCfg<DR>::SMEM) != cudaSuccess)
      return MLA_ERR_CUDA;
    attr_set[dev] = true;
  }
  return launch_pdl(tc_decode_kernel<DR>, dim3(2 * p.G), dim3(DEC_THREADS), (size_t)DecCfg<DR>::SMEM, s, tk, tkr,
                    tqr, tql, p);
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

  CUtensorMap tk, tkr, tqr, tql;
  {
    const uint64_t rows = (uint64_t)std::max<int64_t>(a.total_rows, 1);
    const uint64_t dims[2] = {(uint64_t)W, rows};
    const uint64_t st[1] = {(uint64_t)W * 2};
    const uint32_t box[2] = {64, DEC_BT};
    if (!encode_tmap_bf16(&tk, const_cast<void*>(a.cache), 2, dims, st, box)) return MLA_ERR_CUDA;
  }
  {
    // latent query columns: boxes of 64 columns x 128 rows, 128-byte swizzle (the A operand layout)
    const uint64_t dims[2] = {(uint64_t)W, (uint64_t)a.batch * a.n_q * a.H};
    const uint64_t st[1] = {(uint64_t)W * 2};
    const uint32_t box[2] = {64, DEC_ROWS};
    if (!encode_tmap_bf16(&tql, const_cast<void*>(a.q_abs), 2, dims, st, box)) return MLA_ERR_CUDA;
  }
  tkr = tk;
  tqr = tk;
  if (a.dr) {
    // rotary columns: boxes of 32 columns, 64-byte swizzle
    {
      const uint64_t rows = (uint64_t)std::max<int64_t>(a.total_rows, 1);
      const uint64_t dims[2] = {(uint64_t)W, rows};
      const uint64_t st[1] = {(uint64_t)W * 2};
      const uint32_t box[2] = {32, DEC_BT};
      if (!encode_tmap_bf16(&tkr, const_cast<void*>(a.cache), 2, dims, st, box, 64)) return MLA_ERR_CUDA;
    }
    {
      const uint64_t dims[2] = {(uint64_t)W, (uint64_t)a.batch * a.n_q * a.H};
      const uint64_t st[1] = {(uint64_t)W * 2};
      const uint32_t box[2] = {32, DEC_ROWS};
      if (!encode_tmap_bf16(&tqr, const_cast<void*>(a.q_abs), 2, dims, st, box, 64)) return MLA_ERR_CUDA;
    }
  }
  int st0 = launch_pdl(decode_plan_kernel, dim3(1), dim3(1024), 0, s, p, const_cast<int32_t*>(p.prefix));
  if (st0) return st0;
  int st = a.dr == 0 ? launch_decode_t<0>(tk, tkr, tqr, tql, p, s) : launch_decode_t<64>(tk, tkr, tqr, tql, p, s);
  if (st) return st;
  // 16 CTAs per block (8 rows each): a split block's merge reads 2-3 partial slots of 256 KB
  return launch_pdl(decode_combine_tc_kernel, dim3((unsigned)t.nblocks, DEC_ROWS / 8), dim3(256), 0, s, p);
}

}  // namespace mla
