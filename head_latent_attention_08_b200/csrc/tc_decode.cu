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
//        576 columns, 256-position tiles by TMA through two 96 KB ring slots), computes S = Q K^T in
//        fp32 into a 256-column TMEM slot with N = 256 MMAs, runs the online softmax in fp32 and hands
//        P (bf16) to the value CTA through distributed shared memory (remote st.async stores counted
//        by the value CTA's barrier), 64 positions at a time, with per-row side data (the factor by
//        which O must be rescaled, and the row maxima at the end of each tile);
//      - the value CTA (rank 1) holds all of O in TMEM, streams the latent columns of the same rows
//        (read a second time, from L2, right after the score CTA brought them in) and accumulates
//        O += P . C with 128 x 256 x 16 MMAs, rescales O rows when told to, adds the row sums up from
//        the P it receives, and writes the result.
//    The scores never leave the score CTA, and they are never rounded below fp32 before the
//    exponential: the hand-over is one-way (P and side data forward, "slot free" back).
//  * The score CTA rescales nothing: P is taken against a reference maximum that moves only when a
//    row's maximum grows by more than 2^8 (exact: numerator and denominator share it); the rare move
//    is passed on with the P of that tile, and the value CTA multiplies its O rows before that P.C.
//  * Work: the (block, 256-position tile) units of all sequences are split evenly over the clusters
//    (persistent). A cluster that covers a whole block writes the normalised result; split blocks
//    leave (O, max, sum) partials that a combine kernel merges.
//  * Loads: one thread keeps about one TMA instruction in flight, so several threads issue them (three
//    in the score CTA, two in the value CTA), and the value CTA fetches 64 positions x 256 columns per
//    instruction (a 3-D box over 64-column groups).
//  * Warp roles (640 threads). Score CTA: warps 0, 2, 3 lane 0 TMA, warp 1 lane 0 QK^T, warps 4-19
//    softmax (warp w: rows 32 (w & 3) .., positions [64 c, 64 c + 64) of each tile, c = (w - 4) >> 2),
//    which also move each block's latent query into TMEM. Value CTA: warps 0 and 3 lane 0 TMA, warp 1
//    lane 0 P.C, warp 2 lane 0 hands P slots back, warps 4-19 rescale O, add the row sums up (16
//    positions of every hand-over each) and write O (warp w: rows 32 (w & 3) .., O columns
//    [128 c, 128 c + 128)).
//  * An e4m3 cache (F8; value = code * cache_scale) keeps the same structure: the score CTA streams
//    128-column boxes and runs QK^T as kind::f8f6f4 MMAs against the query split into e4m3 high and
//    low parts (per-row power-of-two scale, both parts in TMEM), and the value CTA stages its units
//    as e4m3 and its rescale warps convert them exactly to f16 for an f16 P.C (P in f16); there the
//    score CTA keeps the row sums and sends them with the maxima.
//  * Every wait is bounded (global-timer limit); a wait that gives up sets the library's status word,
//    and the CTA abandons its work: it issues nothing more, drains its own TMA loads, MMAs and bulk
//    copies and leaves through the cluster barrier.
#include <math.h>
#include <stddef.h>

#include <algorithm>

#include "sm100.cuh"
#include "tc.cuh"

namespace mla {

using namespace sm100;

constexpr int DEC_BT = 256;        // positions per score tile (the N of each QK^T MMA)
constexpr int DEC_HT = 64;         // positions per P hand-over
constexpr int DEC_QT = DEC_BT / DEC_HT;   // hand-overs per tile
constexpr int DEC_THREADS = 640;   // 4 control warps + 16 softmax (score CTA) or rescale/epilogue (value CTA)
constexpr int DEC_SW = 16;         // softmax / epilogue warps
constexpr int DEC_DC = 512;        // latent width handled by this kernel
constexpr int DEC_ROWS = 128;      // rows per block
constexpr int DEC_NPH = 6;         // P hand-over slots in the value CTA (at most)
constexpr int DEC_NPROD = 3;       // TMA-issuing threads of the score CTA
constexpr float DEC_MOVE = 8.f;    // the reference maximum moves when a row maximum exceeds it by 2^8
constexpr int DEC_SMEM_LIMIT = 232448;   // dynamic shared memory per CTA (227 KB)
constexpr int DEC_BAR_BYTES = 4096;

__host__ __device__ constexpr int dec_round1024(int x) { return (x + 1023) / 1024 * 1024; }
__host__ __device__ constexpr int dec_max(int a, int b) { return a > b ? a : b; }

// F8: the cache holds e4m3 codes (one byte per value). The score CTA then streams 128-column boxes
// (still 128-byte rows) and runs QK^T as e4m3 MMAs against a query split into e4m3 high and low parts;
// the value CTA stages its 256-column units as e4m3 and converts them to bf16 (exactly) for P.C.
template <int DR, bool F8 = false>
struct DecCfg {
  static constexpr int DATA_LIMIT = DEC_SMEM_LIMIT - 1024 - DEC_BAR_BYTES;   // 1 KB for alignment
  static constexpr int BOXW = F8 ? 128 : 64;               // cache columns per box (128-byte rows)
  static constexpr int NB_LAT = DEC_DC / BOXW;             // latent boxes of a cache row
  static constexpr int NB = NB_LAT + (DR ? 1 : 0);         // + the rotary box (e4m3: half past the row,
                                                           // read as zeros)
  static constexpr int PARTS = (NB + 2) / 3;               // ring uses per tile
  static constexpr int BOX = DEC_BT * 128;                 // 256 positions x 128 bytes: 32 KB
  // score CTA
  static constexpr int S_OFF_QR = 0;                       // rotary query [128 rows x 128 B]
  static constexpr int S_QR = DR ? DEC_ROWS * 128 : 0;
  static constexpr int S_OFF_RED = S_OFF_QR + S_QR;        // row maxima [2][4][128], row sums [4][128],
                                                           // query maxima [4][128]
  static constexpr int S_OFF_K = dec_round1024(S_OFF_RED + 16 * DEC_ROWS * 4);
  static constexpr int SUPER = 3 * BOX;                    // ring slot: three boxes (12 MMAs per wait)
  static constexpr int NK = (DATA_LIMIT - S_OFF_K) / SUPER;  // ring slots
  // value CTA
  static constexpr int PH = DEC_ROWS * 128;                // P of a hand-over: 128 rows x 64 positions bf16
  static constexpr int SIDE = 4 * 512;                     // side data of a hand-over: 4 quarters x 512 B
  static constexpr int PSLOT = PH + SIDE;                  // 18 KB (a multiple of 1024)
  // bytes that land in a P slot for hand-over cg of a tile: P, then per warp a 16-byte header (the
  // flag), the row factors on the tile's first hand-over and the row maxima on its last (read at the
  // last tile of a block segment), over an e4m3 cache the row sums with them. (With a bf16 cache the
  // value CTA's rescale warps add the row sums up from the P slots themselves; the value CTA of the
  // e4m3 path is bound by its shared-memory traffic, so there the score CTA keeps them.)
  static __host__ __device__ constexpr uint32_t slot_tx(int cg) {
    return (uint32_t)(PH + 4 * (16 + (cg == 0 ? 128 : 0) + (cg == DEC_QT - 1 ? (F8 ? 256 : 128) : 0)));
  }
  static constexpr int NPH = DEC_NPH;                      // P slots
  static constexpr int V_OFF_P = 0;
  static constexpr int V_OFF_V = dec_round1024(NPH * PSLOT);
  static constexpr int UNIT = DEC_HT * 512;                // 64 positions x 256 latent columns bf16: 32 KB
  static constexpr int FUNIT = DEC_HT * 256;               // the same in e4m3: 16 KB
  static constexpr int NV = F8 ? 2 : (DATA_LIMIT - V_OFF_V) / UNIT;   // bf16 (e4m3 cache: f16) value slots
  static constexpr int V_OFF_F = V_OFF_V + NV * UNIT;      // e4m3 staging slots
  static constexpr int NF = F8 ? (DATA_LIMIT - V_OFF_F) / FUNIT : 0;
  static constexpr int OFF_BAR = dec_max(S_OFF_K + NK * SUPER, V_OFF_F + NF * FUNIT);
  static constexpr int SMEM = OFF_BAR + DEC_BAR_BYTES + 1024;
  static_assert(PSLOT % 1024 == 0, "P slots must keep the 1024-byte swizzle alignment");
  static_assert(NPH >= DEC_QT && NPH <= DEC_NPH, "P slots");
  static_assert(NK >= 2, "the cache ring needs two slots");
  static_assert(NV >= 2, "the value ring needs two slots");
  static_assert(!F8 || NF >= 2, "the e4m3 staging ring needs two slots");
  static_assert(!F8 || NF <= 4, "barrier block");
  static_assert(SMEM <= DEC_SMEM_LIMIT, "shared memory budget");
};

// side data of one warp's 32 rows for one half tile (512 B, the layout both CTAs use)
struct DecSide {
  int flag;          // some row of these 32 moved its reference maximum at this tile
  int pad[3];
  float alpha[32];   // factor for O of each row (1 where the reference did not move)
  float m[32];       // reference maximum (log2 units) after this tile
  float l[32];       // e4m3 cache: row sum after this tile (whole row at the last tile of a block)
  float pad2[28];
};
static_assert(sizeof(DecSide) == 512, "side record size");

template <int NK, int NV, int NF>
struct DecBars {
  // score CTA
  uint64_t k_full[NK], k_empty[NK];
  uint64_t qr_full, q_tm, q_empty;
  uint64_t s_full, s_empty;       // the S slot: computed (QK^T commit) / read out (softmax warps)
  uint64_t p_empty[DEC_NPH];      // arrived by the value CTA: a P slot may be written again
  // value CTA
  uint64_t v_full[NV], v_empty[NV];   // (e4m3 cache: v_full = converted to bf16 by the rescale warps)
  uint64_t f_full[NF > 0 ? NF : 1], f_empty[NF > 0 ? NF : 1];   // e4m3 staging slots
  uint64_t p_full[DEC_NPH];       // P + side data landed (transaction count of the bulk copies)
  uint64_t pfree[DEC_NPH];        // P.C read the slot and the rescale/epilogue warps read its side data
  uint64_t o_fix, fix_done;       // rescale hand-shake (one phase per rescale)
  uint64_t o_fin, o_free;         // epilogue hand-shake (one phase per block segment)
  float lsum[4][DEC_ROWS];        // the rescale warps' partial row sums at a segment's end
  // both
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort_flag;
};

struct DecParams {
  const __nv_bfloat16* q_abs;  // [q_rows][W]
  const __nv_bfloat16* cache;  // [total_rows][W]
  int64_t q_rows;
  int W;
  const int32_t* cu;
  int32_t batch, n_q, H, nbps, nblocks;
  int64_t total_rows;
  int causal;
  float scale_log2;           // kq_scale * log2(e)
  const int32_t* prefix;      // [nblocks + 1] exclusive prefix of tiles per block (unless uniform)
  int uniform_tiles;          // > 0: every block has this many tiles (prefix[k] = k * uniform_tiles)
  int G;                      // clusters
  float* out_lat;
  __nv_bfloat16* out16;        // non-null: out_lat is written here in bf16 instead (whole blocks, combine)
  float* lse;
  float* o_part;              // [2G][128][512]
  float* m_part;              // [2G][128] reference maxima (log2 domain)
  float* l_part;              // [2G][128] sums
  int* status;
  unsigned long long wait_ns;
  float cache_scale;          // e4m3 cache: value = code * cache_scale
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 8 x 8 transpose of 16-byte chunks inside each group of eight lanes: before, lane 8 G + i holds in
// c[0..7] the eight chunks of one row i of its group; after, c[t] holds chunk i of row t of the group.
// Three butterfly stages (lane distance 4, 2, 1), each swapping the off-diagonal half of the chunks
// with the partner lane. The map is its own inverse. It turns one-row-per-lane data (the TMEM
// 32x32b layout) into stores where eight lanes cover 128 contiguous bytes of a row, and back for loads.
__device__ __forceinline__ void group8_transpose(uint4 (&c)[8], int lane) {
#pragma unroll
  for (int k = 4; k >= 1; k >>= 1) {
    const bool up = (lane & k) != 0;
#pragma unroll
    for (int lo = 0; lo < 8; ++lo) {
      if (lo & k) continue;
      const int hi = lo | k;
      uint4 v = up ? c[lo] : c[hi];
      v.x = __shfl_xor_sync(0xffffffffu, v.x, k);
      v.y = __shfl_xor_sync(0xffffffffu, v.y, k);
      v.z = __shfl_xor_sync(0xffffffffu, v.z, k);
      v.w = __shfl_xor_sync(0xffffffffu, v.w, k);
      if (up) c[lo] = v; else c[hi] = v;
    }
  }
}

// four e4m3 codes (consecutive bytes of x) -> four f16 values (exact: every e4m3 value is an f16 value)
__device__ __forceinline__ uint2 e4m3x4_to_f16x4(uint32_t x) {
  const __half2_raw h0 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(x & 0xFFFFu), __NV_E4M3);
  const __half2_raw h1 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(x >> 16), __NV_E4M3);
  return make_uint2((uint32_t)h0.x | ((uint32_t)h0.y << 16), (uint32_t)h1.x | ((uint32_t)h1.y << 16));
}

// eight bf16 values (v) times a power of two (p2) as e4m3 high and low parts: hi = e4m3(x),
// lo = e4m3(x - hi), so that hi + lo is x to about 2^-8 relative (both rounded to nearest, saturating);
// four codes per 32-bit word in element order
__device__ __forceinline__ void e4m3_split8(uint4 v, float p2, uint32_t& h0, uint32_t& h1, uint32_t& l0,
                                            uint32_t& l1) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t hs[4], ls[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = make_float2(__uint_as_float(w[e] << 16) * p2, __uint_as_float(w[e] & 0xFFFF0000u) * p2);
    const __nv_fp8x2_storage_t h = __nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(h, __NV_E4M3);
    const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hr));
    const __nv_fp8x2_storage_t l =
        __nv_cvt_float2_to_fp8x2(make_float2(f.x - hf.x, f.y - hf.y), __NV_SATFINITE, __NV_E4M3);
    hs[e] = h;
    ls[e] = l;
  }
  h0 = hs[0] | (hs[1] << 16); h1 = hs[2] | (hs[3] << 16);
  l0 = ls[0] | (ls[1] << 16); l1 = ls[2] | (ls[3] << 16);
}

__device__ __forceinline__ float bf16x8_absmax(uint4 v, float m) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e)
    m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w[e] << 16)), fabsf(__uint_as_float(w[e] & 0xFFFF0000u))));
  return m;
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

// exclusive prefix of tiles per block
__device__ __forceinline__ int64_t dec_prefix(const DecParams& p, int k) {
  return p.uniform_tiles > 0 ? (int64_t)k * p.uniform_tiles : (int64_t)p.prefix[k];
}

// largest k with prefix[k] <= u (the non-empty block that holds unit u, u < prefix[n])
__device__ __forceinline__ int find_block(const DecParams& p, int64_t u) {
  if (p.uniform_tiles > 0) return (int)(u / p.uniform_tiles);
  int lo = 0, hi = p.nblocks - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int64_t)p.prefix[mid] <= u) lo = mid; else hi = mid - 1;
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
    k = u0 < u1 ? find_block(p, u0) : 0;
  }
  __device__ bool next(const DecParams& p, DecSeg& s) {
    if (u >= u1) return false;
    const int64_t bstart = dec_prefix(p, k), bend = dec_prefix(p, k + 1);
    const int64_t send = u1 < bend ? u1 : bend;
    s.k = k;
    s.b = k / p.nbps;
    s.rb = k % p.nbps;
    s.tile0 = (int)(u - bstart);
    s.ntl = (int)(send - u);
    s.complete = (u == bstart) && (send == bend);
    seq_bounds(p, s.b, s.sstart, s.T);
    u = send;
    if (u < u1) k = find_block(p, u);
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
template <int DR, bool F8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(DEC_THREADS, 1)
    tc_decode_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                     const __grid_constant__ CUtensorMap tq, DecParams p) {
  using Cfg = DecCfg<DR, F8>;
  constexpr int NK = Cfg::NK;
  constexpr int NV = Cfg::NV;
  constexpr int NF = Cfg::NF;
  constexpr int NB = Cfg::NB;
  constexpr int NPH = Cfg::NPH;
  using Bars = DecBars<NK, NV, NF>;
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
        mbar_init(&bars->k_full[s], DEC_NPROD);   // every producer arrives once per slot use
        mbar_init(&bars->k_empty[s], 1);
      }
      mbar_init(&bars->qr_full, 1);
      mbar_init(&bars->q_tm, DEC_SW);     // one arrival per softmax warp (each writes its share of Q)
      mbar_init(&bars->q_empty, 1);
      mbar_init(&bars->s_full, 1);
      mbar_init(&bars->s_empty, DEC_SW);  // every softmax warp has read its part of the slot
      for (int s = 0; s < NPH; ++s) mbar_init(&bars->p_empty[s], 1);
    } else {
      for (int s = 0; s < NV; ++s) {
        mbar_init(&bars->v_full[s], F8 ? DEC_SW : 1);   // e4m3: one arrival per converting warp
        mbar_init(&bars->v_empty[s], 1);
      }
      for (int s = 0; s < NF; ++s) {
        mbar_init(&bars->f_full[s], 1);
        mbar_init(&bars->f_empty[s], DEC_SW);
      }
      for (int s = 0; s < NPH; ++s) {
        mbar_init(&bars->p_full[s], 1);
        mbar_init(&bars->pfree[s], DEC_SW + 1);   // the P.C commit and the rescale / epilogue warps
      }
      // arm the first use of every P slot (hand-over s): one local arrival plus the score CTA's stores
      for (int s = 0; s < NPH; ++s) mbar_arrive_expect_tx(&bars->p_full[s], Cfg::slot_tx(s % DEC_QT));
      mbar_init(&bars->o_fix, 1);
      mbar_init(&bars->fix_done, DEC_SW);
      mbar_init(&bars->o_fin, 1);
      mbar_init(&bars->o_free, DEC_SW);

    }
    mbar_init(&bars->drain[0], 1);
    mbar_init(&bars->drain[1], 1);
    bars->abort_flag = 0;
    fence_mbar_init();
    if (scorer) {
      prefetch_tmap(&tk);
      prefetch_tmap(&tq);
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

  const int64_t U = dec_prefix(p, p.nblocks);
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
    const uint32_t tS = tmem + 256;      // columns [256, 512): the 256-position S slot
    uint8_t* sQR = smem + Cfg::S_OFF_QR;
    uint8_t* sK = smem + Cfg::S_OFF_K;
    if ((warp == 0 || warp == 2 || warp == 3) && lane == 0) {
      // ------------------------------- TMA producers -------------------------------
      // One thread keeps about one TMA instruction in flight at a time, so three threads (warps 0, 2
      // and 3) fill the ring together: a ring slot holds three 32 KB boxes, box b of every slot use is
      // loaded by producer b, and each producer arrives once per use (with its bytes, or without a box).
      // A 256-position tile takes three uses: 64-column groups {0, 1, 2}, {3, 4, 5} and {6, 7, 8
      // (rotary)}. The latent query does not pass through the ring (the softmax warps read it), so the
      // cache stream runs on across block boundaries.
      const int pid = warp == 0 ? 0 : warp - 1;
      DecWalk w;
      w.begin(p, u0, u1);
      DecSeg sg;
      int64_t n = 0;          // ring slot uses walked
      int segi = 0, qr_loads = 0;
      bool ok = true;
      auto take_slot = [&](int64_t use) -> int {
        const int s = (int)(use % NK);
        if (use >= NK && !wait_bar(&bars->k_empty[s], (uint32_t)((use / NK) - 1) & 1u)) return -1;
        return s;
      };
      while (ok && w.next(p, sg)) {
        const int qrow = (int)((int64_t)sg.b * p.n_q * p.H + (int64_t)sg.rb * DEC_ROWS);
        if (DR && !F8 && pid == 0) {
          // the rotary query of this segment, once the previous segment's last QK^T has read the old one
          if (segi > 0 && !wait_bar(&bars->q_empty, (uint32_t)(segi - 1) & 1u)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars->qr_full, DEC_ROWS * 128);
          tma_load_2d(sQR, &tq, &bars->qr_full, DEC_DC, qrow);
          ++qr_loads;
        }
        for (int tt = 0; tt < sg.ntl && ok; ++tt) {
          const int y = (int)(sg.sstart + (int64_t)(sg.tile0 + tt) * DEC_BT);
          for (int part = 0; part < Cfg::PARTS; ++part, ++n) {
            const int s = take_slot(n);
            if (s < 0) { ok = false; break; }
            const int j = 3 * part + pid;           // column box of the cache row
            if (j < NB) {
              mbar_arrive_expect_tx(&bars->k_full[s], Cfg::BOX);
              tma_load_2d(sK + s * Cfg::SUPER + pid * Cfg::BOX, &tk, &bars->k_full[s], Cfg::BOXW * j, y);
            } else {
              mbar_arrive(&bars->k_full[s]);
            }
          }
        }
        ++segi;
      }
      if (*abort_flag) {
        // drain the loads in flight before the shared memory is released
        for (int64_t i = (n > NK ? n - NK : 0); i < n; ++i)
          (void)mbar_wait(&bars->k_full[i % NK], (uint32_t)(i / NK) & 1u, drain_ns, p.status);
        if (qr_loads > 0) (void)mbar_wait(&bars->qr_full, (uint32_t)(qr_loads - 1) & 1u, drain_ns, p.status);
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------- QK^T issuer -------------------------------
      // S = Q K^T over the tile's 256 positions: latent groups from the TMEM query (A) and the cache
      // boxes (B, K-major), the rotary group from the shared-memory query. A ring slot (three groups,
      // twelve MMAs) is released by one commit as soon as its MMAs complete; the next tile's QK^T waits
      // only for the softmax warps to have read the S slot out.
      constexpr uint32_t idesc = idesc_bf16_f32(128, DEC_BT, false, false);
      constexpr uint32_t idesc8 = idesc_e4m3_f32(128, DEC_BT);
      const uint64_t kd0 = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t qd0 = smem_desc_sw128(smem_u32(sQR), 16, 1024);
      DecWalk w;
      w.begin(p, u0, u1);
      DecSeg sg;
      int64_t n = 0, g = 0;
      int segi = 0;
      bool ok = true;
      while (ok && w.next(p, sg)) {
        if (!wait_bar(&bars->q_tm, (uint32_t)segi & 1u)) { ok = false; break; }
        if (DR && !F8 && !wait_bar(&bars->qr_full, (uint32_t)segi & 1u)) { ok = false; break; }
        for (int tt = 0; tt < sg.ntl; ++tt, ++g) {
          if (g >= 1 && !wait_bar(&bars->s_empty, (uint32_t)(g - 1) & 1u)) { ok = false; break; }
          tc_fence_after();
          for (int part = 0; part < Cfg::PARTS; ++part, ++n) {
            const int s = (int)(n % NK);
            if (!wait_bar(&bars->k_full[s], (uint32_t)(n / NK) & 1u)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int b = 0; b < 3; ++b) {
              const int j = 3 * part + b;
              if (j >= NB) break;
              const uint64_t kd = kd0 + (uint64_t)((s * Cfg::SUPER + b * Cfg::BOX) >> 4);
              if constexpr (F8) {
                // e4m3: K = 32 per MMA; the query's high part (TMEM columns [0, 128)) and low part
                // (columns [128, 256)) against the same codes; the rotary tile holds the high part in bytes
                // 0..63 of each row and the low part in bytes 64..127
                if (j < Cfg::NB_LAT) {
#pragma unroll
                  for (int kk = 0; kk < 4; ++kk) {
                    mma_e4m3_ts(tS, tQ + j * 32 + kk * 8, kd + (uint64_t)(kk * 2), idesc8, (j | kk) ? 1u : 0u);
                    mma_e4m3_ts(tS, tQ + 128 + j * 32 + kk * 8, kd + (uint64_t)(kk * 2), idesc8, 1u);
                  }
                } else {
#pragma unroll
                  for (int kk = 0; kk < 2; ++kk) {
                    mma_e4m3_ss(tS, qd0 + (uint64_t)(kk * 2), kd + (uint64_t)(kk * 2), idesc8, 1u);
                    mma_e4m3_ss(tS, qd0 + (uint64_t)((kk + 2) * 2), kd + (uint64_t)(kk * 2), idesc8, 1u);
                  }
                }
              } else if (j < 8) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_bf16_ts(tS, tQ + j * 32 + kk * 8, kd + (uint64_t)(kk * 2), idesc, (j | kk) ? 1u : 0u);
              } else {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_bf16_ss(tS, qd0 + (uint64_t)(kk * 2), kd + (uint64_t)(kk * 2), idesc, 1u);
              }
            }
            mma_commit(&bars->k_empty[s]);
          }
          if (!ok) break;
          mma_commit(&bars->s_full);
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
      // warp (q, cg): rows 32 q .. 32 q + 31 (TMEM lanes), positions [64 cg, 64 cg + 64) of each tile;
      // it also moves query columns [128 cg, 128 cg + 128) of each block into TMEM.
      // Its P (32 rows x 64 positions, bf16) and side data go straight into the value CTA's P slot of
      // hand-over 4 g + cg with asynchronous remote stores that count on that slot's barrier.
      const int w16 = warp - 4, q = warp & 3, cg = w16 >> 2;
      const int row = q * 32 + lane;
      const uint32_t lane_off = (uint32_t)(q * 32) << 16;
      float* red = reinterpret_cast<float*>(smem + Cfg::S_OFF_RED);   // maxima [2][4][128], sums [4][128]
      const uint32_t p_remote = map_to_cta(smem_u32(smem + Cfg::V_OFF_P), 1);
      const uint32_t pf_remote = map_to_cta(smem_u32(&bars->p_full[0]), 1);
      DecWalk w;
      w.begin(p, u0, u1);
      DecSeg sg;
      int64_t g = 0;
      int segi = 0;
      while (w.next(p, sg)) {
        // ---- the block's latent query into TMEM: rows 32 q .., latent columns [128 cg, 128 cg + 128),
        // read from global memory (eight lanes per 128-byte row piece, then a lane-group transpose gives
        // every lane its own row), once the previous segment's last QK^T has read the old query. Rows
        // past the end of q_abs read as zeros.
        float sl2 = p.scale_log2;       // score -> log2-domain logit
        if (segi > 0) (void)wait_bar(&bars->q_empty, (uint32_t)(segi - 1) & 1u);
        const int64_t r0 = (int64_t)sg.b * p.n_q * p.H + (int64_t)sg.rb * DEC_ROWS + q * 32 + (lane & ~7);
        // the row pieces of half bx (latent columns 128 cg + 64 bx ..) for the lane's group, transposed
        auto load_half = [&](int bx, uint4 (&c8)[8]) {
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const int64_t rr = r0 + t;
            c8[t] = rr < p.q_rows ? __ldg(reinterpret_cast<const uint4*>(p.q_abs + rr * p.W + cg * 128 + bx * 64 +
                                                                        8 * (lane & 7)))
                                  : make_uint4(0u, 0u, 0u, 0u);
          }
        };
        // all sixteen loads of a lane are issued before any is used
        uint4 ch[2][8];
        load_half(0, ch[0]);
        load_half(1, ch[1]);
        group8_transpose(ch[0], lane);
        group8_transpose(ch[1], lane);
        if constexpr (!F8) {
#pragma unroll
          for (int bx = 0; bx < 2; ++bx) {
            uint32_t r[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              r[4 * c] = ch[bx][c].x; r[4 * c + 1] = ch[bx][c].y; r[4 * c + 2] = ch[bx][c].z; r[4 * c + 3] = ch[bx][c].w;
            }
            tmem_st32(tQ + lane_off + cg * 64 + bx * 32, r);
          }
          tmem_wait_st();
          tc_fence_before();
        } else {
          // e4m3 cache: the row times a power of two p2 (its largest magnitude lands in (224, 448]) as
          // e4m3 high and low parts; latent high part into TMEM columns [32 cg, 32 cg + 32), low part
          // 128 columns further; the warp's 16 rotary columns [16 cg, 16 cg + 16) into the rotary tile
          // (high: 16-byte chunk cg of the row, low: chunk 4 + cg, swizzled). The scores are then in
          // units of 1 / p2 / cache_scale.
          const int64_t own = r0 - (lane & ~7) + lane;
          uint4 rp[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
          if (DR && own < p.q_rows) {
            const uint4* src = reinterpret_cast<const uint4*>(p.q_abs + own * p.W + DEC_DC + 16 * cg);
            rp[0] = __ldg(src);
            rp[1] = __ldg(src + 1);
          }
          float amax = bf16x8_absmax(rp[1], bf16x8_absmax(rp[0], 0.f));
#pragma unroll
          for (int bx = 0; bx < 2; ++bx)
#pragma unroll
            for (int c = 0; c < 8; ++c) amax = bf16x8_absmax(ch[bx][c], amax);
          float* qmx = red + 12 * DEC_ROWS;
          qmx[cg * DEC_ROWS + row] = amax;
          named_bar_sync(1 + q, 128);         // the four warps of these rows
          const float rmax = fmaxf(fmaxf(qmx[row], qmx[DEC_ROWS + row]), fmaxf(qmx[2 * DEC_ROWS + row], qmx[3 * DEC_ROWS + row]));
          // largest power of two p2 with rmax * p2 <= 448 (kept within the normal range)
          const float p2 = rmax > 0.f ? __uint_as_float(__float_as_uint(fminf(448.f / rmax, 0x1p100f)) & 0x7F800000u)
                                      : 1.f;
          sl2 = p.scale_log2 * p.cache_scale / p2;
          // the pieces again (now from L2), half by half, to keep registers for the split
#pragma unroll 1
          for (int bx = 0; bx < 2; ++bx) {
            uint4 c8[8];
            load_half(bx, c8);
            group8_transpose(c8, lane);
            uint32_t hi[16], lo[16];
#pragma unroll
            for (int c = 0; c < 8; ++c) e4m3_split8(c8[c], p2, hi[2 * c], hi[2 * c + 1], lo[2 * c], lo[2 * c + 1]);
            tmem_st16(tQ + lane_off + cg * 32 + bx * 16, hi);
            tmem_st16(tQ + lane_off + 128 + cg * 32 + bx * 16, lo);
          }
          if (DR) {
            uint4 h, lw;
            e4m3_split8(rp[0], p2, h.x, h.y, lw.x, lw.y);
            e4m3_split8(rp[1], p2, h.z, h.w, lw.z, lw.w);
            uint8_t* qrow = sQR + row * 128;
            *reinterpret_cast<uint4*>(qrow + ((cg ^ (row & 7)) << 4)) = h;
            *reinterpret_cast<uint4*>(qrow + (((4 + cg) ^ (row & 7)) << 4)) = lw;
            fence_proxy_async_smem();   // generic stores read by the MMAs (async proxy)
          }
          tmem_wait_st();
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->q_tm);
        const int cnt = row_count(sg.T, p.n_q, p.H, sg.rb * DEC_ROWS + row, p.causal);
        float m_ref = -INFINITY, l = 0.f;   // (l: e4m3 cache only)
        for (int tt = 0; tt < sg.ntl; ++tt, ++g) {
          const bool last = tt + 1 == sg.ntl;
          float s[64];
          (void)wait_bar(&bars->s_full, (uint32_t)g & 1u);
          tc_fence_after();
          {
            uint32_t r0[32], r1[32];
            tmem_ld32(tS + lane_off + cg * 64, r0);
            tmem_ld32(tS + lane_off + cg * 64 + 32, r1);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              s[c] = __uint_as_float(r0[c]);
              s[32 + c] = __uint_as_float(r1[c]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0 && !*abort_flag) mbar_arrive(&bars->s_empty);
          // mask (only where the tile crosses the row's limit) and the raw row maximum
          const int t0 = (sg.tile0 + tt) * DEC_BT + cg * 64;
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
          float* mx = red + (g & 1) * 4 * DEC_ROWS;
          mx[cg * DEC_ROWS + row] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
          named_bar_sync(1 + q, 128);         // the four warps of these rows
          const float mx_t = fmaxf(fmaxf(mx[row], mx[DEC_ROWS + row]), fmaxf(mx[2 * DEC_ROWS + row], mx[3 * DEC_ROWS + row])) *
                             sl2;             // the scale is positive: the order is kept
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
          // the P slot of this hand-over must have been handed back by the value CTA
          const int64_t i = (int64_t)DEC_QT * g + cg;
          const int hs = (int)(i % NPH);
          if (i >= NPH) (void)wait_bar(&bars->p_empty[hs], (uint32_t)((i / NPH) - 1) & 1u);
          const bool send = !*abort_flag;
          const uint32_t dst = p_remote + (uint32_t)(hs * Cfg::PSLOT);
          const uint32_t bar = pf_remote + (uint32_t)(hs * 8);
          const uint32_t prow = dst + (uint32_t)(row * 128);
          // P in bf16 (round to nearest even), 8 positions (16 bytes, one swizzled chunk of the row) at a
          // time; the value CTA adds the row sums up from the same stored values. Over an e4m3 cache P is
          // f16 (the type of the converted codes; 11 bits) and the row sum, of the unrounded values, is
          // kept here.
          float sum = 0.f;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = ex2(fmaf(s[8 * c + 2 * e], sl2, -mu)), x1 = ex2(fmaf(s[8 * c + 2 * e + 1], sl2, -mu));
              if constexpr (F8) {
                const __half2 h2 = __floats2half2_rn(x0, x1);
                pk[e] = *reinterpret_cast<const uint32_t*>(&h2);
                sum += x0 + x1;
              } else {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(x0, x1);
                pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
              }
            }
            if (send) st_async_v4(prow + (uint32_t)((c ^ (lane & 7)) * 16), make_uint4(pk[0], pk[1], pk[2], pk[3]), bar);
          }
          float lsend = 0.f;
          if constexpr (F8) {
            l += sum;
            lsend = l;
            if (last) {
              // the block's row sum is the sum of the four warps' sums: the last warp of the row sends it
              float* ls = red + 8 * DEC_ROWS;
              ls[cg * DEC_ROWS + row] = l;
              named_bar_sync(1 + q, 128);
              if (cg == DEC_QT - 1)
                lsend = (ls[row] + ls[DEC_ROWS + row]) + (ls[2 * DEC_ROWS + row] + ls[3 * DEC_ROWS + row]);
            }
          }
          const int flag = (cg == 0) ? (__any_sync(0xffffffffu, moved) ? 1 : 0) : 0;
          // side data in 16-byte stores: the flag on every hand-over, the row factors on the tile's
          // first, the maxima on its last (the value CTA reads them at a segment's end)
          const uint32_t sd = dst + (uint32_t)(Cfg::PH + q * 512);
          const int src4 = (4 * lane) & 31;     // lanes 0..7 gather rows 4 lane .. 4 lane + 3
          if (send && lane == 0) st_async_v4(sd + offsetof(DecSide, flag), make_uint4((uint32_t)flag, 0u, 0u, 0u), bar);
          if (cg == 0) {
            uint4 v;
            v.x = __float_as_uint(__shfl_sync(0xffffffffu, alpha, src4));
            v.y = __float_as_uint(__shfl_sync(0xffffffffu, alpha, src4 + 1));
            v.z = __float_as_uint(__shfl_sync(0xffffffffu, alpha, src4 + 2));
            v.w = __float_as_uint(__shfl_sync(0xffffffffu, alpha, src4 + 3));
            if (send && lane < 8) st_async_v4(sd + offsetof(DecSide, alpha) + 16 * lane, v, bar);
          }
          if (cg == DEC_QT - 1) {
            uint4 vm;
            vm.x = __float_as_uint(__shfl_sync(0xffffffffu, m_ref, src4));
            vm.y = __float_as_uint(__shfl_sync(0xffffffffu, m_ref, src4 + 1));
            vm.z = __float_as_uint(__shfl_sync(0xffffffffu, m_ref, src4 + 2));
            vm.w = __float_as_uint(__shfl_sync(0xffffffffu, m_ref, src4 + 3));
            if (send && lane < 8) st_async_v4(sd + offsetof(DecSide, m) + 16 * lane, vm, bar);
            if constexpr (F8) {
              uint4 vl;
              vl.x = __float_as_uint(__shfl_sync(0xffffffffu, lsend, src4));
              vl.y = __float_as_uint(__shfl_sync(0xffffffffu, lsend, src4 + 1));
              vl.z = __float_as_uint(__shfl_sync(0xffffffffu, lsend, src4 + 2));
              vl.w = __float_as_uint(__shfl_sync(0xffffffffu, lsend, src4 + 3));
              if (send && lane < 8) st_async_v4(sd + offsetof(DecSide, l) + 16 * lane, vl, bar);
            }
          }
        }
        ++segi;
      }
    }
  } else {
    // =========================================================================================
    // value CTA
    // =========================================================================================
    const uint32_t tO = tmem;   // all 512 columns
    uint8_t* sP = smem + Cfg::V_OFF_P;
    uint8_t* sV = smem + Cfg::V_OFF_V;
    uint8_t* sF = smem + Cfg::V_OFF_F;
    if ((warp == 0 || warp == 3) && lane == 0) {
      // ------------------------------- TMA producers -------------------------------
      // per hand-over (64 positions): two value slot uses of 256 latent columns, each one TMA
      // instruction of four 64-column groups (a 3-D box: columns within a group, positions, groups);
      // use m is issued by producer m % 2 (warps 0 and 3: two instructions in flight). An e4m3 cache
      // goes to the staging slots instead (two 128-column groups per instruction, unswizzled), which
      // the rescale warps convert into the value slots.
      const int pid = warp == 0 ? 0 : 1;
      DecWalk w;
      w.begin(p, u0, u1);
      DecSeg sg;
      int64_t n = 0;          // value slot uses walked
      bool ok = true;
      while (ok && w.next(p, sg)) {
        for (int tt = 0; tt < sg.ntl && ok; ++tt) {
          for (int cg = 0; cg < DEC_QT && ok; ++cg) {
            const int y = (int)(sg.sstart + (int64_t)(sg.tile0 + tt) * DEC_BT + cg * DEC_HT);
            for (int nh = 0; nh < 2; ++nh, ++n) {
              if ((n & 1) != pid) continue;
              if constexpr (F8) {
                const int f = (int)(n % NF);
                if (n >= NF && !wait_bar(&bars->f_empty[f], (uint32_t)((n / NF) - 1) & 1u)) { ok = false; break; }
                mbar_arrive_expect_tx(&bars->f_full[f], Cfg::FUNIT);
                tma_load_3d(sF + f * Cfg::FUNIT, &tv, &bars->f_full[f], 0, y, 2 * nh);
                continue;
              }
              const int s = (int)(n % NV);
              if (n >= NV && !wait_bar(&bars->v_empty[s], (uint32_t)((n / NV) - 1) & 1u)) { ok = false; break; }
              mbar_arrive_expect_tx(&bars->v_full[s], Cfg::UNIT);
              tma_load_3d(sV + s * Cfg::UNIT, &tv, &bars->v_full[s], 0, y, 4 * nh);
            }
          }
        }
      }
      if (*abort_flag) {
        if constexpr (F8) {
          for (int64_t i = (n > NF ? n - NF : 0); i < n; ++i)
            if ((i & 1) == pid) (void)mbar_wait(&bars->f_full[i % NF], (uint32_t)(i / NF) & 1u, drain_ns, p.status);
        } else {
          for (int64_t i = (n > NV ? n - NV : 0); i < n; ++i)
            if ((i & 1) == pid) (void)mbar_wait(&bars->v_full[i % NV], (uint32_t)(i / NV) & 1u, drain_ns, p.status);
        }
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------- P.C issuer -------------------------------
      // O[:, 256 nh + ...] += P (128 x 64, K-major, from the P slot) . C (64 x 256, MN-major, from a
      // value slot); each value slot is released by its own commit
      // (f16 operands over an e4m3 cache)
      constexpr uint32_t idesc = F8 ? idesc_f16_f32(128, 256, false, true) : idesc_bf16_f32(128, 256, false, true);
      const uint64_t pd0 = smem_desc_sw128(smem_u32(sP), 16, 1024);
      const uint64_t vd0 = smem_desc_sw128(smem_u32(sV), DEC_HT * 128, 1024);
      DecWalk w;
      w.begin(p, u0, u1);
      DecSeg sg;
      int64_t i = 0;
      int segi = 0, fixes = 0;
      bool ok = true;
      while (ok && w.next(p, sg)) {
        for (int tt = 0; tt < sg.ntl && ok; ++tt) {
          for (int cg = 0; cg < DEC_QT; ++cg, ++i) {
            const int hs = (int)(i % NPH);
            if (!wait_bar(&bars->p_full[hs], (uint32_t)(i / NPH) & 1u)) { ok = false; break; }
            const bool first = tt == 0 && cg == 0;
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
            fence_proxy_async_smem();   // P was stored by the peer's threads: order it before the MMAs read it
            const uint64_t pd = pd0 + (uint64_t)((hs * Cfg::PSLOT) >> 4);
            for (int nh = 0; nh < 2; ++nh) {
              const int64_t vu = 2 * i + nh;
              const int s = (int)(vu % NV);
              if (!wait_bar(&bars->v_full[s], (uint32_t)(vu / NV) & 1u)) { ok = false; break; }
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
            if (tt + 1 == sg.ntl && cg == DEC_QT - 1) mma_commit(&bars->o_fin);
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
      // once P.C of a hand-over has completed and the rescale / epilogue warps have read its side data:
      // re-arm the P slot's landing barrier for its next use, then tell the score CTA it may write it
      const uint32_t pe_remote = map_to_cta(smem_u32(&bars->p_empty[0]), 0);
      DecWalk w;
      w.begin(p, u0, u1);
      DecSeg sg;
      int64_t total = 0;
      while (w.next(p, sg)) total += (int64_t)DEC_QT * sg.ntl;
      int64_t i = 0;
      for (; i < total; ++i) {
        const int hs = (int)(i % NPH);
        if (!wait_bar(&bars->pfree[hs], (uint32_t)(i / NPH) & 1u)) break;
        if (i + NPH < total) {
          mbar_arrive_expect_tx(&bars->p_full[hs], Cfg::slot_tx((int)((i + NPH) % DEC_QT)));
          mbar_arrive_remote_release(pe_remote + (uint32_t)(hs * 8));
        }
      }
      if (*abort_flag) {
        // abandoned work: the score CTA may still have remote stores in flight into the slots that are
        // armed; wait (bounded) for each armed hand-over to land before this CTA may leave
        for (int64_t u = i; u < total && u < i + NPH; ++u)
          (void)mbar_wait(&bars->p_full[u % NPH], (uint32_t)(u / NPH) & 1u, drain_ns, p.status);
      }
    } else if (warp >= 4) {
      // ------------------------------- rescale and epilogue -------------------------------
      // warp (q, cv): rows 32 q .. 32 q + 31, O columns [128 cv, 128 cv + 128)
      const int w16 = warp - 4, q = warp & 3, cv = w16 >> 2;
      const int row = q * 32 + lane;
      const uint32_t lane_off = (uint32_t)(q * 32) << 16;
      const uint32_t tcol = tO + lane_off + cv * 128;
      // e4m3 cache: value use u from its staging slot into a value slot as f16 (the codes, exactly),
      // each warp 64 of the 1024 16-byte chunks ([group 2][position 64][chunk 8]); a chunk's 16 codes
      // are 16 columns of a 64-column f16 group, two swizzled 16-byte chunks of the position's row.
      // 16-byte accesses go out eight lanes at a time: the eight lanes of each phase take chunks 0..3 of
      // one position and 4..7 of the next (or the reverse), so that both the staging reads (unswizzled)
      // and the stores (opposite position parities) touch eight different bank quads.
      auto convert_use = [&](int64_t u) {
        const int fs = (int)(u % (NF > 0 ? NF : 1)), vs = (int)(u % NV);
        bool ok = wait_bar(&bars->f_full[fs], (uint32_t)(u / (NF > 0 ? NF : 1)) & 1u);
        if (ok && u >= NV) ok = wait_bar(&bars->v_empty[vs], (uint32_t)((u / NV) - 1) & 1u);
        if (!ok) return;
        const uint8_t* src = sF + fs * Cfg::FUNIT;
        uint8_t* dstu = sV + vs * Cfg::UNIT;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int base = w16 * 64 + e * 32;
          const int k = (lane >> 2) & 1;
          const int g = base >> 9, pos = ((base >> 3) & 63) + 2 * ((lane >> 4) & 1) + k;
          const int c16 = 4 * (k ^ ((lane >> 3) & 1)) + (lane & 3);
          const int id = (g << 9) | (pos << 3) | c16;
          const uint4 v = *reinterpret_cast<const uint4*>(src + id * 16);
          const uint2 a = e4m3x4_to_f16x4(v.x), b = e4m3x4_to_f16x4(v.y);
          const uint2 c = e4m3x4_to_f16x4(v.z), d = e4m3x4_to_f16x4(v.w);
          const int cb = (c16 & 3) * 2;
          uint8_t* rowp = dstu + (2 * g + (c16 >> 2)) * (DEC_HT * 128) + pos * 128;
          *reinterpret_cast<uint4*>(rowp + ((cb ^ (pos & 7)) << 4)) = make_uint4(a.x, a.y, b.x, b.y);
          *reinterpret_cast<uint4*>(rowp + (((cb + 1) ^ (pos & 7)) << 4)) = make_uint4(c.x, c.y, d.x, d.y);
        }
        fence_proxy_async_smem();   // generic stores read by the P.C MMAs (async proxy)
        __syncwarp();
        if (lane == 0 && !*abort_flag) {
          mbar_arrive(&bars->f_empty[fs]);
          mbar_arrive(&bars->v_full[vs]);
        }
      };
      DecWalk w;
      w.begin(p, u0, u1);
      DecSeg sg;
      int64_t i = 0;
      int segi = 0, fixes = 0;
      while (w.next(p, sg)) {
        float lp = 0.f;   // the row's sum over positions 16 cv .. 16 cv + 15 of every hand-over so far
        for (int tt = 0; tt < sg.ntl; ++tt) {
          for (int cg = 0; cg < DEC_QT; ++cg, ++i) {
            const int hs = (int)(i % NPH);
            if constexpr (F8) {
              convert_use(2 * i);
              convert_use(2 * i + 1);
            }
            (void)wait_bar(&bars->p_full[hs], (uint32_t)(i / NPH) & 1u);
            const DecSide* sd = reinterpret_cast<const DecSide*>(sP + hs * Cfg::PSLOT + Cfg::PH);
            const int any = sd[0].flag | sd[1].flag | sd[2].flag | sd[3].flag;
            if (any) {
              const bool ok = wait_bar(&bars->o_fix, (uint32_t)fixes & 1u);
              ++fixes;
              tc_fence_after();
              if (ok && sd[q].flag) {
                const float alpha = sd[q].alpha[lane];
#pragma unroll 1
                for (int cc = 0; cc < 128; cc += 32) {
                  uint32_t r[32];
                  tmem_ld32(tcol + cc, r);
                  tmem_wait_ld();
#pragma unroll
                  for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
                  tmem_st32(tcol + cc, r);
                }
                tmem_wait_st();
              }
              if (sd[q].flag) lp *= sd[q].alpha[lane];   // the row sum follows the reference as O does
              tc_fence_before();
              __syncwarp();
              if (lane == 0 && !*abort_flag) mbar_arrive(&bars->fix_done);
            }
            if constexpr (!F8) {
              // this hand-over's P (the values the P.C MMAs read), positions 16 cv .. 16 cv + 15 of the
              // row (two swizzled 16-byte chunks), into the row sum
              const uint8_t* prow = sP + hs * Cfg::PSLOT + row * 128;
              const uint4 pa = *reinterpret_cast<const uint4*>(prow + (((2 * cv) ^ (row & 7)) << 4));
              const uint4 pb = *reinterpret_cast<const uint4*>(prow + (((2 * cv + 1) ^ (row & 7)) << 4));
              const uint32_t pw[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
              float ps = 0.f;
#pragma unroll
              for (int e = 0; e < 8; ++e) ps += __uint_as_float(pw[e] << 16) + __uint_as_float(pw[e] & 0xFFFF0000u);
              lp += ps;
            }
            if (tt + 1 == sg.ntl && cg == DEC_QT - 1) {
              // ---- epilogue of the segment: O / l (whole block) or the partial (O, m, l)
              const float m_ref = sd[q].m[lane];
              // the row sum: the four warps' parts of the row, added in a fixed order (e4m3 cache: sent
              // by the score CTA)
              float ltot;
              if constexpr (F8) {
                ltot = sd[q].l[lane];
              } else {
                bars->lsum[cv][row] = lp;
                named_bar_sync(1 + q, 128);
                ltot = (bars->lsum[0][row] + bars->lsum[1][row]) + (bars->lsum[2][row] + bars->lsum[3][row]);
              }
              const bool ok = wait_bar(&bars->o_fin, (uint32_t)segi & 1u);
              tc_fence_after();
              const int ri = sg.rb * DEC_ROWS + row;
              const int rows_seq = p.n_q * p.H;
              const int64_t orow = (int64_t)sg.b * rows_seq + ri;
              const int slotp = 2 * pair + (segi == 0 ? 0 : 1);
              const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
              const float mul = (sg.complete ? inv : 1.f) * (F8 ? p.cache_scale : 1.f);
              float* dst = sg.complete ? p.out_lat + orow * DEC_DC : p.o_part + ((int64_t)slotp * DEC_ROWS + row) * DEC_DC;
              // each lane scales its own row; after the lane-group transpose, store t of a lane goes to
              // row 8 (lane / 8) + t of the warp's rows, columns 4 (lane % 8) .. of the 32 just read, so
              // eight lanes write 128 contiguous bytes of one row
              const int gfirst = q * 32 + (lane & ~7);               // first row of the lane's group
              float* gdst = dst + (int64_t)(gfirst - row) * DEC_DC + cv * 128 + 4 * (lane & 7);
              const bool bf_out = sg.complete && p.out16 != nullptr;
              __nv_bfloat16* g16 = bf_out ? p.out16 + ((int64_t)sg.b * rows_seq + sg.rb * DEC_ROWS + gfirst) * DEC_DC +
                                                cv * 128 + 4 * (lane & 7)
                                          : nullptr;
              const int grows = !ok ? 0 : (sg.complete ? min(8, rows_seq - (sg.rb * DEC_ROWS + gfirst)) : 8);
#pragma unroll 1
              for (int cc = 0; cc < 128; cc += 32) {
                uint32_t r[32];
                tmem_ld32(tcol + cc, r);
                tmem_wait_ld();
                uint4 ch[8];
#pragma unroll
                for (int c = 0; c < 8; ++c)
                  ch[c] = make_uint4(__float_as_uint(__uint_as_float(r[4 * c]) * mul),
                                     __float_as_uint(__uint_as_float(r[4 * c + 1]) * mul),
                                     __float_as_uint(__uint_as_float(r[4 * c + 2]) * mul),
                                     __float_as_uint(__uint_as_float(r[4 * c + 3]) * mul));
                group8_transpose(ch, lane);
                if (bf_out) {
                  // bf16 out_lat: eight lanes write 64 contiguous bytes of a row
#pragma unroll
                  for (int t = 0; t < 8; ++t) {
                    const __nv_bfloat162 lo = __floats2bfloat162_rn(__uint_as_float(ch[t].x), __uint_as_float(ch[t].y));
                    const __nv_bfloat162 hi = __floats2bfloat162_rn(__uint_as_float(ch[t].z), __uint_as_float(ch[t].w));
                    if (t < grows)
                      *reinterpret_cast<uint2*>(g16 + (int64_t)t * DEC_DC + cc) =
                          make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
                  }
                } else {
#pragma unroll
                  for (int t = 0; t < 8; ++t)
                    if (t < grows) *reinterpret_cast<uint4*>(gdst + (int64_t)t * DEC_DC + cc) = ch[t];
                }
              }
              if (ok && cv == 0) {
                if (sg.complete) {
                  if (ri < rows_seq && p.lse)
                    p.lse[orow] = ltot > 0.f ? (m_ref + log2f(ltot)) * 0.69314718055994531f : -INFINITY;
                } else {
                  p.m_part[(int64_t)slotp * DEC_ROWS + row] = m_ref;
                  p.l_part[(int64_t)slotp * DEC_ROWS + row] = ltot;
                }
              }
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
  cluster_sync();     // the score CTA stores nothing into the value CTA after this point
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------------------
// combine: 16 CTAs per block, eight rows each (a warp per row, four float4 of the 512 latent columns per
// lane); merges the partials of blocks split across clusters and writes zeros / -inf for blocks with
// nothing to attend to. A lane's loads for one partial slot are independent of each other and of the
// next slot's, so several are in flight at once.
// ---------------------------------------------------------------------------------------------
constexpr int DEC_CB_ROWS = 8;   // rows per combine CTA

__global__ void __launch_bounds__(256) decode_combine_tc_kernel(DecParams p) {
  __shared__ int slots[256];
  __shared__ float wts[DEC_CB_ROWS][256];
  __shared__ int nsl;
  griddep_wait();
  griddep_launch_dependents();
  const int k = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y * DEC_CB_ROWS + warp;           // row within the block
  const int64_t bstart = dec_prefix(p, k), bend = dec_prefix(p, k + 1);
  const int b = k / p.nbps, rb = k % p.nbps;
  const int rows_seq = p.n_q * p.H;
  const int ri = rb * DEC_ROWS + r;
  const bool row_ok = ri < rows_seq;
  const int64_t orow = (int64_t)b * rows_seq + ri;
  float4* dst = reinterpret_cast<float4*>(p.out_lat + orow * DEC_DC);
  uint2* dst16 = p.out16 ? reinterpret_cast<uint2*>(p.out16 + orow * DEC_DC) : nullptr;
  // four consecutive out_lat values (a float4) at float4 index j of the row, in the output's type
  auto put = [&](int j, float4 v) {
    if (dst16) {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
      dst16[j] = make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
    } else {
      dst[j] = v;
    }
  };
  if (bend == bstart) {
    if (row_ok) {
#pragma unroll
      for (int j = 0; j < 4; ++j) put(lane + 32 * j, make_float4(0.f, 0.f, 0.f, 0.f));
      if (lane == 0 && p.lse) p.lse[orow] = -INFINITY;
    }
    return;
  }
  const int64_t U = dec_prefix(p, p.nblocks);
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
  if (!row_ok) return;
  const int n = nsl;
  // the row's weights w_i = 2^(m_i - M) and its sum L (slots in index order: the sum does not depend
  // on timing)
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
  float4 acc[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
  for (int i = 0; i < n; ++i) {
    const float w = wts[warp][i];
    const float4* src = reinterpret_cast<const float4*>(p.o_part + ((int64_t)slots[i] * DEC_ROWS + r) * DEC_DC);
    float4 o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) o[j] = src[lane + 32 * j];
    if (w != 0.f) {   // (a slot with no visible position is not used)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc[j].x = fmaf(w, o[j].x, acc[j].x); acc[j].y = fmaf(w, o[j].y, acc[j].y);
        acc[j].z = fmaf(w, o[j].z, acc[j].z); acc[j].w = fmaf(w, o[j].w, acc[j].w);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) put(lane + 32 * j, make_float4(acc[j].x * inv, acc[j].y * inv, acc[j].z * inv, acc[j].w * inv));
  if (lane == 0 && p.lse) p.lse[orow] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
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
  // an e4m3 cache is read by TMA from a 16-byte aligned base (rows of 576 or 512 bytes)
  if (a.cache_f8 && (reinterpret_cast<uintptr_t>(a.cache) & 15u)) return false;
  return nblocks < (1LL << 31) / tiles;
}

struct TcDecodePlan {
  int nbps, nblocks, G;
  size_t off_prefix, off_o, off_m, off_l, total;
};

template <int DR, bool F8>
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
  cfg.dynamicSmemBytes = DecCfg<DR, F8>::SMEM;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaFuncSetAttribute(tc_decode_kernel<DR, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       DecCfg<DR, F8>::SMEM);
  const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, (void*)tc_decode_kernel<DR, F8>, &cfg);
  if (e != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = sm_count() / 2;
  }
  return n;
}

// clusters of two CTAs that can be resident at once (the kernel is persistent: more would run as a
// second wave); computed once per device and tile variant
static int max_active_clusters(int dr, bool f8) {
  static int cached[64][4] = {{0}};
  const int dev = current_device();
  const int v = (dr == 0 ? 0 : 1) + (f8 ? 2 : 0);
  if (dev < 0 || dev >= 64) return sm_count() / 2;
  if (cached[dev][v] == 0)
    cached[dev][v] = v == 0 ? max_active_clusters_t<0, false>() : v == 1 ? max_active_clusters_t<64, false>()
                   : v == 2 ? max_active_clusters_t<0, true>() : max_active_clusters_t<64, true>();
  return cached[dev][v];
}

static TcDecodePlan plan_tc(const DecodeArgs& a) {
  TcDecodePlan t;
  t.nbps = (int)ceil_div((int64_t)a.n_q * a.H, DEC_ROWS);
  t.nblocks = a.batch * t.nbps;
  const int64_t units_max = (int64_t)t.nblocks * std::max<int64_t>(1, ceil_div(a.max_seqlen, DEC_BT));
  const int maxc = max_active_clusters(a.dr, a.cache_f8);
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

template <int DR, bool F8>
static int launch_decode_t(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                           const DecParams& p, cudaStream_t s) {
  static bool attr_set[64] = {false};
  const int dev = current_device();
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(tc_decode_kernel<DR, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DecCfg<DR, F8>::SMEM) != cudaSuccess)
      return MLA_ERR_CUDA;
    attr_set[dev] = true;
  }
  return launch_pdl(tc_decode_kernel<DR, F8>, dim3(2 * p.G), dim3(DEC_THREADS), (size_t)DecCfg<DR, F8>::SMEM, s,
                    tk, tv, tq, p);
}

int tc_decode_launch(const DecodeArgs& a, cudaStream_t s) {
  const TcDecodePlan t = plan_tc(a);
  const int W = a.dc + a.dr;
  char* ws = static_cast<char*>(a.workspace);
  DecParams p{};
  p.q_abs = static_cast<const __nv_bfloat16*>(a.q_abs);
  p.cache = static_cast<const __nv_bfloat16*>(a.cache);
  p.q_rows = (int64_t)a.batch * a.n_q * a.H;
  p.W = W;
  p.cu = a.cu_seqlens; p.batch = a.batch; p.n_q = a.n_q; p.H = a.H; p.nbps = t.nbps; p.nblocks = t.nblocks;
  p.total_rows = a.total_rows; p.causal = a.causal ? 1 : 0;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.cache_scale = a.cache_f8 ? a.cache_scale : 1.f;
  p.prefix = reinterpret_cast<int32_t*>(ws + t.off_prefix);
  p.G = t.G;
  p.out_lat = a.out_lat; p.lse = a.lse;
  p.out16 = static_cast<__nv_bfloat16*>(a.out_lat_bf16);
  p.o_part = reinterpret_cast<float*>(ws + t.off_o);
  p.m_part = reinterpret_cast<float*>(ws + t.off_m);
  p.l_part = reinterpret_cast<float*>(ws + t.off_l);
  p.status = device_status_ptr();
  p.wait_ns = (unsigned long long)wait_limit();
  if (!p.status) return MLA_ERR_CUDA;
  if (t.nblocks == 0) return MLA_OK;

  // the cache: 128-position boxes of 64 columns for the score CTA, 64-position x 256-column boxes for
  // the value CTA; the query: 128 rows x 64 columns. All 128-byte swizzled (the MMA operand layout).
  CUtensorMap tk, tv, tq;
  const uint64_t rows = (uint64_t)std::max<int64_t>(a.total_rows, 1);
  if (a.cache_f8) {
    // e4m3: 256-position x 128-column boxes for the score CTA (the rotary box starts at column 512 and
    // reads its last 64 columns as zeros), 64-position x 256-column unswizzled staging boxes (two
    // 128-column groups) for the value CTA
    {
      const uint64_t dims[2] = {(uint64_t)W, rows};
      const uint64_t st[1] = {(uint64_t)W};
      const uint32_t box[2] = {128, DEC_BT};
      if (!encode_tmap_u8(&tk, const_cast<void*>(a.cache), 2, dims, st, box, 128)) return MLA_ERR_CUDA;
    }
    {
      const uint64_t dims[3] = {128, rows, (uint64_t)(a.dc / 128)};
      const uint64_t st[2] = {(uint64_t)W, 128};
      const uint32_t box[3] = {128, DEC_HT, 2};
      if (!encode_tmap_u8(&tv, const_cast<void*>(a.cache), 3, dims, st, box, 0)) return MLA_ERR_CUDA;
    }
  } else {
    {
      const uint64_t dims[2] = {(uint64_t)W, rows};
      const uint64_t st[1] = {(uint64_t)W * 2};
      const uint32_t box[2] = {64, DEC_BT};
      if (!encode_tmap_bf16(&tk, const_cast<void*>(a.cache), 2, dims, st, box)) return MLA_ERR_CUDA;
    }
    {
      // positions step by a row, groups by 64 columns: one box is 64 positions x 256 columns, laid out
      // as four 64-column groups of [64 positions x 128 B] (the MN-major B operand of P.C)
      const uint64_t dims[3] = {64, rows, (uint64_t)(W / 64)};
      const uint64_t st[2] = {(uint64_t)W * 2, 128};
      const uint32_t box[3] = {64, DEC_HT, 4};
      if (!encode_tmap_bf16(&tv, const_cast<void*>(a.cache), 3, dims, st, box)) return MLA_ERR_CUDA;
    }
  }
  {
    const uint64_t dims[2] = {(uint64_t)W, (uint64_t)a.batch * a.n_q * a.H};
    const uint64_t st[1] = {(uint64_t)W * 2};
    const uint32_t box[2] = {64, DEC_ROWS};
    if (!encode_tmap_bf16(&tq, const_cast<void*>(a.q_abs), 2, dims, st, box)) return MLA_ERR_CUDA;
  }
  // Equal-length sequences (total_rows = batch * max_seqlen with every T_b <= max_seqlen), each block
  // reading up to the sequence's last position: every block has the same tile count, known here, and
  // the plan kernel is not needed. With one cluster per block on top, every block is written whole by
  // its cluster, and nothing is left to combine.
  const bool equal_blocks = a.total_rows == (int64_t)a.batch * a.max_seqlen && (!a.causal || t.nbps == 1);
  if (equal_blocks && a.max_seqlen > 0) {
    p.uniform_tiles = (int)ceil_div(a.max_seqlen, DEC_BT);
  } else {
    const int st0 = launch_pdl(decode_plan_kernel, dim3(1), dim3(1024), 0, s, p, const_cast<int32_t*>(p.prefix));
    if (st0) return st0;
  }
  int st = a.cache_f8 ? (a.dr == 0 ? launch_decode_t<0, true>(tk, tv, tq, p, s)
                                    : launch_decode_t<64, true>(tk, tv, tq, p, s))
                       : (a.dr == 0 ? launch_decode_t<0, false>(tk, tv, tq, p, s)
                                    : launch_decode_t<64, false>(tk, tv, tq, p, s));
  if (st) return st;
  if (equal_blocks && t.G == t.nblocks && a.max_seqlen > 0) return MLA_OK;
  // 16 CTAs per block (eight rows each): a split block's merge reads its partial slots of 256 KB
  return launch_pdl(decode_combine_tc_kernel, dim3((unsigned)t.nblocks, DEC_ROWS / DEC_CB_ROWS), dim3(256), 0, s, p);
}

}  // namespace mla
