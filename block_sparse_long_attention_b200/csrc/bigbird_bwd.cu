// Backward pass of BigBird ITC block-sparse attention for B200 (sm_100a).
//
// Gradients of sum(dout * out) with respect to q, k and v for the same block
// pattern as the forward [TFG-BigBird, section "BigBird：从二次方注意力到线性稀疏注意力";
// HF-Pegasus, section "三类注意力组合"], by the chain rule through each row's
// softmax: with p = exp(s - lse) recomputed from the forward's row
// log-sum-exp and D = rowsum(dout * out),
//   dp = dout v^T,  ds = p (dp - D),
//   dq = ds k / sqrt(d),  dk = ds^T q / sqrt(d),  dv = p^T dout.
//
// Four launches, in stream order (the dq kernel as the dk/dv kernel's
// programmatic dependent, free to start on the SMs the dk/dv kernel leaves,
// as it needs nothing the dk/dv kernel writes; the dk/dv kernel, whose units
// are the larger, goes first so that the finer dq units fill the end),
// nothing accumulated with atomics (the gradients are the same bit for bit
// on every run):
//   1. bwd_rowdot_kernel: D = rowsum(dout * out) into the workspace;
//   2. bwd_kernel<true> (dk, dv): key-stationary. A unit is 128 key rows (key
//      blocks j, j+1, or the two global key blocks against one range of query
//      tiles) against the query tiles that attend either block -- the pattern
//      transposed, found by scanning rand_attn (a long list goes out in
//      chunks). Per query tile: S^T = K Q^T and dP^T = V dO^T, P^T and dS^T by
//      one thread per key row (the query's lse and D from shared memory), then
//      dV += P^T dO and dK += dS^T Q (two TS-MMAs);
//   3. bwd_kernel<false> (dq): query-stationary. A unit is the forward's: 128
//      query rows (query blocks i, i+1, or the two global blocks against one
//      range of key tiles) against a list of 64-key tiles. Per key tile:
//      S = Q K^T and dP = dO V^T (tcgen05 SS-MMAs, M = 128, N = 64, K = 64,
//      fp32 in TMEM), P and dS by one thread per query row (bf16, written
//      back over the S and dP columns), then dQ += dS K (TS-MMA, dS from TMEM,
//      K as loaded, d contiguous);
//   4. bwd_sum_kernel: the global rows' dq and the global key blocks' dk, dv
//      are split over ranges; their partial sums (workspace) are added here,
//      all three in one launch.
//
// Both attention kernels are persistent (2 CTAs per SM, 256 TMEM columns:
// S | dP | accumulator 1 | accumulator 2) and warp-specialised: warps 0-7 the
// elementwise part and the epilogue (two warps per row, 32 columns each),
// warp 8 TMA, warps 9 and 11 the MMAs (one thread each: S and its product,
// dP and its product), warp 10 unit preparation and
// scheduling (tickets from a workspace counter, reset by the CTA that
// finishes last). Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "../../include/bigbird_attn.h"
#include "bb_internal.h"
#include "sm100_ptx.cuh"

namespace bbw {

using namespace bb;

constexpr int kBlock = 64;     // tokens per tile: a block of 64, or half a block of 128
constexpr int kRows = 128;     // stationary rows per unit (two tiles)
constexpr int kMaxList = 42;   // moving tiles per unit chunk
constexpr int kMaxR = 16;
constexpr int kSplit = 8;      // tiles per range of a global unit
constexpr int kThreads = 384;  // warps 0-7 elementwise, 8 TMA, 9 and 11 MMA, 10 prep
constexpr int kElemWarps = 8;
constexpr uint32_t kChunkBytes = kBlock * 64 * 2;  // 64 rows x 64 columns bf16: one TMA box
// TMEM columns: S (or S^T) of a step, 64 fp32 columns, then P_hi and P_lo
// (bf16 pairs) over them; dP (or dP^T) in the next 64, then dS_hi and dS_lo
// (BGeo::x_col gives the S columns of each buffer); the accumulators:
constexpr uint32_t kColA1 = 128;  // dQ, or dV: d fp32 columns; dK follows

// Sizes that follow from the head dimension d (64 or 128): a row of d values
// is cut into d / 64 chunks (chunk c of a 64-row tile at c * 8 KB, of the
// unit's 128 stationary rows at c * 16 KB). At d = 64 two CTAs share an SM
// (256 TMEM columns each; more shared memory is requested than used so that a
// third never waits for TMEM); at d = 128 the two stationary operands alone
// take 64 KB, so one CTA per SM (512 TMEM columns for dk/dv: S | dP | dV | dK).
template <int kD>
struct BGeo {
  static constexpr int kChunks = kD / 64;
  static constexpr uint32_t kTileBytes = kBlock * kD * 2;
  static constexpr uint32_t kAChunkBytes = kRows * 64 * 2;
  static constexpr int kCtasPerSm = kD == 64 ? 2 : 1;
  static constexpr uint32_t kColA2 = kColA1 + kD;
  // At d = 128 (one CTA per SM) S and dP are double-buffered: step g uses
  // buffer g % 2, the second pair in the columns after the accumulators, so
  // the next step's S and dP are computed while the elementwise warps work on
  // this one; the moving-tile ring is then three deep (a stage stays in use
  // until the previous step's gradient MMAs are complete).
  static constexpr int kBufs = kD == 128 ? 2 : 1;
  static constexpr int kStages = kD == 128 ? 3 : 2;
  __host__ __device__ static constexpr uint32_t tmem_cols(bool) { return kD == 64 ? 256u : 512u; }
  // S (X) columns of buffer b; dP (Y) follow at + 64
  __host__ __device__ static constexpr uint32_t x_col(uint32_t b, bool kv) { return b == 0 ? 0u : (kv ? 384u : 256u); }
};
constexpr int kSmemRequest64 = 112 * 1024;

constexpr uint32_t kStatusBadRandAttn = 1u;
constexpr uint32_t kStatusTimeout = 2u;

// Workspace: counters (ints) [0] dq tickets, [1] dq CTAs done, [2] dk/dv
// tickets, [3] dk/dv CTAs done; then D [B*H*L] fp32; then the partial sums.
constexpr size_t kCounterBytes = 256;

// One unit chunk: stationary tiles `top` (rows 0..63) and `bot` (rows 64..127,
// or -1) of head bh against `n` moving tiles.
struct Unit {
  int32_t n;
  int32_t bh;
  int32_t top, bot;
  int32_t split;   // partial-sum slot of a split global unit, or -1
  int32_t first;   // 1: the unit's first chunk (accumulators start from zero)
  int32_t last;    // 1: the unit's last chunk (epilogue follows)
  int32_t stop;    // 1: no more units for this CTA
  int32_t mt[kMaxList];    // moving tiles
  uint64_t vm[kMaxList];   // dq kernel: validity bits of the moving (key) tile
  uint8_t hm[kMaxList];    // bit 0: rows 0..63 use the tile, bit 1: rows 64..127
};

struct Params {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const uint16_t* dout;
  const float* lse;       // [B*H*L] natural log
  const float* dd;        // D [B*H*L]
  const int32_t* rand_attn;
  const uint8_t* seq_mask;
  float* g1;              // dq (dq kernel) or dv (dk/dv kernel), [B*H*L, d]
  float* g2;              // dk (dk/dv kernel)
  float* part1;           // partial sums of split global units [BH, nparts, 128, d] (g1)
  float* part2;           // ... (g2)
  int* counters;          // this kernel's [tickets, done]
  uint32_t* status;
  int H, L, nb, r, BH;
  int nt;                 // 64-token tiles per sequence
  int sparse;
  int nsplit;             // ranges per global unit (1: write the gradient directly)
  int n_glob;             // global units per range: 1 (block 64: both global blocks) or 2 (block 128)
  int nparts;             // n_glob * nsplit
  int n_mid_per_head;     // middle units per head
  int n_mid_units;
  int total_units;
  float scale_log2;       // log2(e) / sqrt(d)
  float bias_raw;         // -10000 sqrt(d): the masked-key bias in units of q.k
  float scale;            // 1 / sqrt(d)
};

// TMA store maps of the gradient tiles at d = 64 ([rows, 64] fp32, boxes of
// 64 rows x 32 columns): the direct outputs g1, g2 and the partial sums.
struct StoreMaps {
  CUtensorMap o1, o2, p1, p2;
};

template <int kD>
struct __align__(1024) Smem {
  uint8_t a1[kRows * kD * 2];                   // Q (dq) or K (dk/dv) of the unit: two tiles
  uint8_t a2[kRows * kD * 2];                   // dO (dq) or V (dk/dv)
  uint8_t b1[BGeo<kD>::kStages][BGeo<kD>::kTileBytes];    // K (dq) or Q (dk/dv) of a step
  uint8_t b2[BGeo<kD>::kStages][BGeo<kD>::kTileBytes];    // V (dq) or dO (dk/dv)
  // d = 64: one fp32 accumulator tile of the unit (four boxes of 64 rows x
  // 32 columns, 128-byte swizzle) on its way out through TMA stores
  uint8_t ostage[kD == 64 ? kRows * 64 * 4 : 1024];
  float col_lse[BGeo<kD>::kStages][kBlock];         // dk/dv: lse and D of the step's query tile
  float col_d[BGeo<kD>::kStages][kBlock];
  Unit unit[4];
  uint64_t info_full[4];
  uint64_t info_empty[4];
  uint64_t a_full, a_free;
  uint64_t b_full[BGeo<kD>::kStages], b_empty[BGeo<kD>::kStages];
  uint64_t x_full[2];     // S and dP of step g are in TMEM buffer g % kBufs
  uint64_t p_full[2];     // P and dS of step g written (elementwise warps)
  uint64_t xy_free[2][2]; // [part][buffer]: a part's gradient MMAs of the step are complete
  uint64_t acc_full;   // a unit's accumulators are complete
  uint64_t acc_free;   // ... and read by the epilogue (4 warps)
  uint64_t stage_free; // d = 64: ostage may be written (the previous tile's stores have read it)
  uint64_t tile_ready; // d = 64: the elementwise warps have written their part of ostage
  uint32_t tmem_base;
  uint32_t rbits[32];  // dk/dv prep: per query block of a scan batch, which key blocks it picked at random
};

__device__ __forceinline__ void flag_timeout(const Params& p) { atomicOr(p.status, kStatusTimeout); }

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16),
// completion counted on the mbarrier in bytes.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// 64 validity bits of key block kb of batch b (bit c: seq_mask != 0).
__device__ __forceinline__ uint64_t key_valid_bits(const uint8_t* seq_mask, int L, int b, int kb) {
  const uint4* src = reinterpret_cast<const uint4*>(seq_mask + static_cast<size_t>(b) * L + static_cast<size_t>(kb) * kBlock);
  uint64_t bits = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 w = __ldg(src + i);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t m = __vcmpne4(ws[j], 0u) & 0x01010101u;  // one bit per byte
      bits |= static_cast<uint64_t>((m * 0x01020408u) >> 24) << (16 * i + 4 * j);
    }
  }
  return bits;
}

// ------------------------------------------------------------ unit building

// Everything is counted in 64-token tiles: a block of 64 is one tile (kBt =
// 1), a block of 128 two (kBt = 2). Unit u of either kernel when its list fits
// one chunk: a global unit (the global rows stacked against one range of 8
// tiles, every row attending every tile: both global blocks in one unit at
// block 64, one unit per global block at block 128), a full-attention unit
// (tiles 2j, 2j+1 against every tile), or -- dq kernel only -- a middle unit:
// query blocks (i, i+1) against the union of their key blocks with a half
// mask per tile (block 64), or query block i against its own key blocks
// (block 128) [TFG-BigBird, section "随机块掩码是如何生成的"; HF-Pegasus,
// section "三类注意力组合"]. In the dk/dv kernel the stationary tiles are key
// tiles and the moving ones query tiles; a global or full-attention unit
// decodes the same way (every query attends a global key block, and in full
// attention every key). Whole warp: the lanes fetch the random entries, lane
// 0 builds the list.
template <int kBt>
__device__ void build_simple(const Params& p, int u, Unit& ui, int lane) {
  int n = 0;
  // one tile, merging the half masks of a tile listed twice (set semantics)
  auto add_tile = [&](int t, int hm) {
    for (int e = 0; e < n; ++e)
      if (ui.mt[e] == t) {
        ui.hm[e] |= static_cast<uint8_t>(hm);
        return;
      }
    ui.mt[n] = t;
    ui.hm[n] = static_cast<uint8_t>(hm);
    ++n;
  };
  // one block of the pattern; an entry outside [0, nb) is skipped and reported
  auto add_block = [&](int kb, int hm) {
    if (kb < 0 || kb >= p.nb) {
      atomicOr(p.status, kStatusBadRandAttn);
      return;
    }
#pragma unroll
    for (int t = 0; t < kBt; ++t) add_tile(kb * kBt + t, hm);
  };
  int bh, top, bot, split = -1;
  if (u >= p.n_mid_units) {
    const int v = u - p.n_mid_units;
    int t0, t1;
    if (p.sparse) {
      bh = v / p.nparts;
      const int part = v % p.nparts;
      const int g = part / p.nsplit;
      const int s = part % p.nsplit;
      if (p.n_glob == 1) {
        top = 0;
        bot = p.nt - 1;
      } else {
        top = g == 0 ? 0 : p.nt - 2;
        bot = top + 1;
      }
      t0 = s * kSplit;
      t1 = min(p.nt, t0 + kSplit);
      split = p.nsplit > 1 ? part : -1;
    } else {
      const int npair = (p.nt + 1) / 2;
      bh = v / npair;
      const int pp = v % npair;
      top = 2 * pp;
      bot = 2 * pp + 1 < p.nt ? 2 * pp + 1 : -1;
      t0 = 0;
      t1 = p.nt;
    }
    if (lane == 0)
      for (int t = t0; t < t1; ++t) add_tile(t, bot >= 0 ? 3 : 1);
  } else {
    bh = u / p.n_mid_per_head;
    const int pp = u % p.n_mid_per_head;
    const int h = bh % p.H;
    if (kBt == 1) {
      const int i = 1 + 2 * pp;
      const bool pair = i + 1 <= p.nb - 2;
      const int both = pair ? 3 : 1;
      const int nrand = pair ? 2 * p.r : p.r;
      const int32_t* ra = p.rand_attn + (static_cast<size_t>(h) * (p.nb - 2) + (i - 1)) * p.r;
      const int rv = lane < nrand ? __ldg(ra + lane) : -1;
      if (lane == 0) {
        add_block(i - 1, 1);
        add_block(i, both);
        add_block(i + 1, both);
        if (pair) add_block(i + 2, 2);
        add_block(0, both);
        add_block(p.nb - 1, both);
      }
      for (int t = 0; t < nrand; ++t) {
        const int x = __shfl_sync(0xffffffffu, rv, t);
        if (lane == 0) add_block(x, t < p.r ? 1 : 2);
      }
      top = i;
      bot = pair ? i + 1 : -1;
    } else {
      const int i = 1 + pp;
      const int32_t* ra = p.rand_attn + (static_cast<size_t>(h) * (p.nb - 2) + (i - 1)) * p.r;
      const int rv = lane < p.r ? __ldg(ra + lane) : -1;
      if (lane == 0) {
        add_block(i - 1, 3);
        add_block(i, 3);
        add_block(i + 1, 3);
        add_block(0, 3);
        add_block(p.nb - 1, 3);
      }
      for (int t = 0; t < p.r; ++t) {
        const int x = __shfl_sync(0xffffffffu, rv, t);
        if (lane == 0) add_block(x, 3);
      }
      top = 2 * i;
      bot = 2 * i + 1;
    }
  }
  if (lane == 0) {
    ui.n = n;
    ui.bh = bh;
    ui.top = top;
    ui.bot = bot;
    ui.split = split;
    ui.first = 1;
    ui.last = 1;
    ui.stop = 0;
  }
}

// ------------------------------------------------------------ preparation

// Unit preparation and scheduling (one warp), up to two chunks ahead: a CTA's
// first unit is its block index, later ones are tickets from the workspace
// counter (units numbered longest first). Publishes a stop slot at the end.
// The dk/dv kernel's middle units -- key blocks (j, j+1) at block 64, key
// block j (two tiles) at block 128 -- list the query tiles of the query
// blocks that attend them: the two global query blocks, the window
// neighbours, and every middle query block whose random entries pick one of
// them, found by scanning rand_attn 32 (block 128: 16) query blocks at a time
// (set semantics: repeated or window-overlapping picks add nothing). A list
// longer than a chunk goes out as several chunks; only the first starts the
// accumulators from zero and only the last is followed by the epilogue.
template <int kD, int kBt, bool kKV>
__device__ void prep_role(Smem<kD>& s, const Params& p) {
  const int lane = threadIdx.x & 31;
  uint32_t ut = 0;  // chunks published so far
  auto acquire = [&]() -> Unit* {
    int ok = 1;
    // at most two chunks ahead: chunk ut - 2 released (which implies ut - 4)
    if (lane == 0) ok = ut < 2 || mbar_wait(smem_u32(&s.info_empty[(ut - 2) & 3]), ((ut - 2) >> 2) & 1);
    if (!__shfl_sync(0xffffffffu, ok, 0)) return nullptr;
    return &s.unit[ut & 3];
  };
  auto finish = [&](Unit& ui) {
    __syncwarp();
    const int n = ui.n;
    const int b = ui.bh / p.H;
    if (!kKV)
      for (int e = lane; e < n; e += 32) ui.vm[e] = p.seq_mask ? key_valid_bits(p.seq_mask, p.L, b, ui.mt[e]) : ~0ull;
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&s.info_full[ut & 3]));
    ++ut;
    // the moving tiles into L2 ahead of the TMA loads
    const size_t row0 = static_cast<size_t>(ui.bh) * p.L;
    for (int t = lane; t < 2 * n; t += 32) {
      const uint16_t* base = t < n ? (kKV ? p.q : p.k) : (kKV ? p.dout : p.v);
      prefetch_l2_bulk(base + (row0 + static_cast<size_t>(ui.mt[t < n ? t : t - n]) * kBlock) * kD,
                       BGeo<kD>::kTileBytes);
    }
  };
  int u = blockIdx.x;
  s.rbits[lane] = 0;
  __syncwarp();
  for (;;) {
    Unit* ui = acquire();
    if (!ui) {
      if (lane == 0) flag_timeout(p);
      return;
    }
    if (u >= p.total_units) {
      if (lane == 0) {
        ui->stop = 1;
        mbar_arrive(smem_u32(&s.info_full[ut & 3]));
      }
      return;
    }
    int next = 0;
    if (lane == 0) next = static_cast<int>(gridDim.x) + atomicAdd(&p.counters[0], 1);
    if (!kKV || u >= p.n_mid_units) {
      build_simple<kBt>(p, u, *ui, lane);
      finish(*ui);
    } else {
      constexpr int kBatch = kBt == 1 ? 32 : 16;  // query blocks per scan batch (kBt tiles each)
      const int bh = u / p.n_mid_per_head;
      const int pp = u % p.n_mid_per_head;
      const int h = bh % p.H;
      // key blocks j and j + 1 (block 64) or key block j (block 128)
      const int j = kBt == 1 ? 1 + 2 * pp : 1 + pp;
      const bool pair = kBt == 1 && j + 1 <= p.nb - 2;
      auto header = [&](Unit& c, int first) {
        if (lane == 0) {
          c.bh = bh;
          c.top = kBt * j;
          c.bot = kBt == 2 ? 2 * j + 1 : (pair ? j + 1 : -1);
          c.split = -1;
          c.first = first;
          c.last = 0;
          c.stop = 0;
        }
      };
      header(*ui, 1);
      int n = 0;
      bool ok = true;
      // at block 128 both tiles of key block j are used by every row of an
      // attending query block: bits 1 and 2 together
      const int jbits = kBt == 1 ? 1 : 3;
      for (int base = 0; base < p.nb && ok; base += kBatch) {
        const int q = base + lane;
        int hm = 0;
        if (lane < kBatch && q < p.nb) {
          if (q == 0 || q == p.nb - 1) {
            hm = kBt == 2 || pair ? 3 : 1;
          } else {
            hm = (abs(q - j) <= 1 ? jbits : 0) | (pair && abs(q - (j + 1)) <= 1 ? 2 : 0);
          }
        }
        // random picks of the middle query blocks qlo .. qhi-1 of this batch
        const int qlo = max(base, 1), qhi = min(base + kBatch, p.nb - 1);
        if (qhi > qlo) {
          const int cnt = (qhi - qlo) * p.r;
          const int32_t* ra = p.rand_attn + (static_cast<size_t>(h) * (p.nb - 2) + (qlo - 1)) * p.r;
          for (int e = lane; e < cnt; e += 32) {
            const int x = __ldg(ra + e);
            if (x < 0 || x >= p.nb) atomicOr(p.status, kStatusBadRandAttn);
            const int bits = (x == j ? jbits : 0) | (pair && x == j + 1 ? 2 : 0);
            // lanes holding entries of the same query block meet here: atomic
            if (bits) atomicOr(&s.rbits[qlo - base + e / p.r], static_cast<unsigned int>(bits));
          }
        }
        __syncwarp();
        hm |= static_cast<int>(s.rbits[lane]);
        __syncwarp();
        s.rbits[lane] = 0;
        __syncwarp();
        const uint32_t mask = __ballot_sync(0xffffffffu, hm != 0);
        const int c = kBt * __popc(mask);  // tiles this batch adds
        if (n + c > kMaxList) {
          if (lane == 0) ui->n = n;
          finish(*ui);
          ui = acquire();
          if (!ui) {
            ok = false;
            break;
          }
          header(*ui, 0);
          n = 0;
        }
        if (hm) {
          const int pos = n + kBt * __popc(mask & ((1u << lane) - 1u));
#pragma unroll
          for (int t = 0; t < kBt; ++t) {
            ui->mt[pos + t] = kBt * q + t;
            ui->hm[pos + t] = static_cast<uint8_t>(hm);
          }
        }
        n += c;
      }
      if (!ok) {
        if (lane == 0) flag_timeout(p);
        return;
      }
      if (lane == 0) {
        ui->n = n;
        ui->last = 1;
      }
      finish(*ui);
    }
    u = __shfl_sync(0xffffffffu, next, 0);
  }
}

// Columns 16q .. 16q+15 of the S / dP tiles (piece q, read by one warp) are
// replaced by that piece's hi terms (columns 16q .. 16q+7, packed pairs) and
// lo terms (16q+8 .. 16q+15).
__device__ __forceinline__ uint32_t hi_col(int q) { return 16 * q; }
__device__ __forceinline__ uint32_t lo_col(int q) { return 16 * q + 8; }

// ------------------------------------------------------------ TMA

// Stationary tiles once per unit (after the previous unit's last S/dP MMAs
// have read them), then the two moving tiles of every step (and, in the dk/dv
// kernel, the query tile's lse and D) into a 2-deep ring.
// dq kernel: A1 = Q, A2 = dO, B1 = K, B2 = V. dk/dv kernel: A1 = K, A2 = V,
// B1 = Q, B2 = dO.
template <int kD, bool kKV>
__device__ void producer_role(Smem<kD>& s, const Params& p, const CUtensorMap* tmA1, const CUtensorMap* tmA2,
                              const CUtensorMap* tmB1, const CUtensorMap* tmB2) {
  using G = BGeo<kD>;
  const int lane = threadIdx.x & 31;
  const uint64_t pol_a = l2_policy_evict_first();
  const uint64_t pol_b = l2_policy_evict_last();
  uint32_t g = 0, ua = 0;
  for (uint32_t ut = 0;; ++ut) {
    if (!warp_wait(smem_u32(&s.info_full[ut & 3]), (ut >> 2) & 1)) {
      if (lane == 0) flag_timeout(p);
      return;
    }
    const Unit& ui = s.unit[ut & 3];
    if (ui.stop) break;
    int ok = 1;
    if (lane == 0) {
      const int32_t row0 = ui.bh * p.L;
      if (ui.first) {
        ok = mbar_wait(smem_u32(&s.a_free), (ua & 1) ^ 1);
        if (ok) {
          const uint32_t bar = smem_u32(&s.a_full);
          mbar_arrive_expect_tx(bar, (ui.bot >= 0 ? 4 : 2) * G::kTileBytes);
          // chunk c of the unit's rows at c * 16 KB: the top tile, then the bottom one
#pragma unroll
          for (int c = 0; c < G::kChunks; ++c) {
            const uint32_t off = c * G::kAChunkBytes;
            tma_load_2d(smem_u32(s.a1) + off, tmA1, bar, 64 * c, row0 + ui.top * kBlock, pol_a);
            tma_load_2d(smem_u32(s.a2) + off, tmA2, bar, 64 * c, row0 + ui.top * kBlock, pol_a);
            if (ui.bot >= 0) {
              tma_load_2d(smem_u32(s.a1) + off + kChunkBytes, tmA1, bar, 64 * c, row0 + ui.bot * kBlock, pol_a);
              tma_load_2d(smem_u32(s.a2) + off + kChunkBytes, tmA2, bar, 64 * c, row0 + ui.bot * kBlock, pol_a);
            }
          }
        }
        ++ua;
      }
      for (int e = 0; e < ui.n && ok; ++e, ++g) {
        const int st = g % BGeo<kD>::kStages;
        ok = mbar_wait(smem_u32(&s.b_empty[st]), ((g / BGeo<kD>::kStages) & 1) ^ 1);
        if (!ok) break;
        const uint32_t bar = smem_u32(&s.b_full[st]);
        const int32_t row = row0 + ui.mt[e] * kBlock;
        mbar_arrive_expect_tx(bar, 2 * G::kTileBytes + (kKV ? 2 * kBlock * 4 : 0));
#pragma unroll
        for (int c = 0; c < G::kChunks; ++c) {
          tma_load_2d(smem_u32(s.b1[st]) + c * kChunkBytes, tmB1, bar, 64 * c, row, pol_b);
          tma_load_2d(smem_u32(s.b2[st]) + c * kChunkBytes, tmB2, bar, 64 * c, row, pol_b);
        }
        if (kKV) {
          bulk_load(smem_u32(s.col_lse[st]), p.lse + row, kBlock * 4, bar);
          bulk_load(smem_u32(s.col_d[st]), p.dd + row, kBlock * 4, bar);
        }
      }
    }
    if (!__shfl_sync(0xffffffffu, ok, 0)) {
      if (lane == 0) flag_timeout(p);
      return;
    }
    g = __shfl_sync(0xffffffffu, g, 0);
    ua = __shfl_sync(0xffffffffu, ua, 0);
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&s.info_empty[ut & 3]));
  }
}

// ------------------------------------------------------------ MMA

// One thread. Per step: X = A1 B1^T, Y = A2 B2^T (SS, M = 128, N = 64,
// K = 64), once the previous step's gradient MMAs have read P and dS out of
// those columns; then, once P and dS are written, the gradient MMAs (TS, A =
// the hi and lo terms from TMEM, B = the moving tile with d contiguous, K =
// 64 moving rows):
//   dq kernel:   acc1 += (dS_hi + dS_lo) B1                          (dQ += dS K)
//   dk/dv kernel: acc1 += (P_hi + P_lo) B2, acc2 += (dS_hi + dS_lo) B1 (dV += P^T dO, dK += dS^T Q)
template <int kD, bool kKV, int kPart>
__device__ void mma_role(Smem<kD>& s, const Params& p, uint32_t tmem) {
  using G = BGeo<kD>;
  constexpr int kSt = G::kStages;
  constexpr int kNB = G::kBufs;
  // Two issuing threads (warps 9 and 11), each with its own products:
  //   dk/dv: part 0 S^T -> dV += P^T dO;  part 1 dP^T -> dK += dS^T Q;
  //   dq:    part 0 S   -> dQ += dS K;     part 1 dP.
  // A part reuses its S or dP columns (buffer g % kNB) once the gradient MMAs
  // that read them, kNB steps back, are complete (dk/dv: its own,
  // xy_free[part]; dq: dP waits for dQ, xy_free[0], while S's columns are
  // read by no MMA and free once P is written). With two buffers a step's S
  // and dP go out before the previous step's gradient MMAs.
  constexpr bool kHasGrad = kKV || kPart == 0;
  const uint32_t idesc1 = idesc_f32acc(kRows, kBlock, true, false);
  const uint32_t idesc2 = idesc_f32acc(kRows, 64, true, true);  // one 64-column chunk of d
  const uint32_t a_src = smem_u32(kPart == 0 ? s.a1 : s.a2);
  // gradient MMAs of step gb (zero: its unit's first step, the accumulator is
  // overwritten once the unit before has been read out, acc_free phase uab;
  // last: its unit's last step), then the moving stage is released
  auto issue_grad = [&](uint32_t gb, bool zero, bool last, uint32_t uab) -> bool {
    const int st = gb % kSt;
    const uint32_t bb = gb % kNB;
    if (kHasGrad) {
      if (zero && !mbar_wait(smem_u32(&s.acc_free), (uab & 1) ^ 1)) return false;
      if (!mbar_wait(smem_u32(&s.p_full[bb]), (gb / kNB) & 1)) return false;
      tc_fence_after();
      const uint32_t b1 = smem_u32(s.b1[st]), b2 = smem_u32(s.b2[st]);
      // dk/dv part 0: dV += (P_hi + P_lo) dO (P in the S columns, B = b2);
      // dk/dv part 1: dK += (dS_hi + dS_lo) Q (dS in the dP columns, B = b1);
      // dq: dQ += (dS_hi + dS_lo) K (dS in the dP columns, B = b1)
      const uint32_t acc = kKV && kPart == 1 ? G::kColA2 : kColA1;
      const uint32_t pcol = G::x_col(bb, kKV) + (kKV && kPart == 0 ? 0u : 64u);
      const uint32_t bsrc = kKV && kPart == 0 ? b2 : b1;
      // accumulator columns 64 c .. 64 c + 63 from chunk c of the moving tile
#pragma unroll
      for (int c = 0; c < G::kChunks; ++c) {
        const uint32_t boff = c * kChunkBytes;
#pragma unroll
        for (int kk = 0; kk < kBlock / 16; ++kk) {
          mma_ts(tmem + acc + 64 * c, tmem + pcol + hi_col(kk), sdesc_sw128(bsrc + boff + kk * 2048, 8192, 1024),
                 idesc2, (zero && kk == 0) ? 0u : 1u);
          mma_ts(tmem + acc + 64 * c, tmem + pcol + lo_col(kk), sdesc_sw128(bsrc + boff + kk * 2048, 8192, 1024),
                 idesc2, 1u);
        }
      }
      mma_commit(smem_u32(&s.xy_free[kPart][bb]));
      if (last) mma_commit(smem_u32(&s.acc_full));
    }
    mma_commit(smem_u32(&s.b_empty[st]));
    return true;
  };
  uint32_t g = 0, ua = 0;
  bool pend = false, pend_zero = false, pend_last = false;
  uint32_t pend_g = 0, pend_ua = 0;
  bool ok = true;
  for (uint32_t ut = 0; ok; ++ut) {
    if (!mbar_wait(smem_u32(&s.info_full[ut & 3]), (ut >> 2) & 1)) { ok = false; break; }
    const Unit& ui = s.unit[ut & 3];
    if (ui.stop) break;
    const int n = ui.n;
    const bool first = ui.first, last = ui.last;
    if (first && !mbar_wait(smem_u32(&s.a_full), ua & 1)) { ok = false; break; }
    for (int e = 0; e < n; ++e, ++g) {
      const int st = g % kSt;
      const uint32_t bb = g % kNB;
      if (!mbar_wait(smem_u32(&s.b_full[st]), (g / kSt) & 1)) { ok = false; break; }
      if (g >= static_cast<uint32_t>(kNB)) {
        const uint32_t ph = ((g / kNB) - 1) & 1;  // step g - kNB
        if (kKV && !mbar_wait(smem_u32(&s.xy_free[kPart][bb]), ph)) { ok = false; break; }
        if (!kKV && kPart == 1 && !mbar_wait(smem_u32(&s.xy_free[0][bb]), ph)) { ok = false; break; }
      }
      tc_fence_after();
      const uint32_t b_src = smem_u32(kPart == 0 ? s.b1[st] : s.b2[st]);
      const uint32_t x_col = G::x_col(bb, kKV) + (kPart == 0 ? 0u : 64u);  // this part's S or dP columns
      // K = d in steps of 16: four per 64-column chunk
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk)
        mma_ss(tmem + x_col, sdesc_sw128(a_src + (kk >> 2) * G::kAChunkBytes + (kk & 3) * 32, 16, 1024),
               sdesc_sw128(b_src + (kk >> 2) * kChunkBytes + (kk & 3) * 32, 16, 1024), idesc1, kk > 0 ? 1u : 0u);
      mma_commit(smem_u32(&s.x_full[bb]));
      if (last && e == n - 1) mma_commit(smem_u32(&s.a_free));
      const bool zero = first && e == 0;
      const bool lst = last && e == n - 1;
      if (kNB == 1) {
        if (!issue_grad(g, zero, lst, ua)) { ok = false; break; }
      } else {
        if (pend && !issue_grad(pend_g, pend_zero, pend_last, pend_ua)) { ok = false; break; }
        pend = true;
        pend_g = g;
        pend_zero = zero;
        pend_last = lst;
        pend_ua = ua;
      }
    }
    if (!ok) break;
    if (first) ++ua;
    mbar_arrive(smem_u32(&s.info_empty[ut & 3]));
  }
  if (ok && pend && !issue_grad(pend_g, pend_zero, pend_last, pend_ua)) ok = false;
  if (!ok) flag_timeout(p);
}

// ------------------------------------------------------------ elementwise

// 16 columns of one row: P = exp2(x scale_log2 + c) with c = bias scale_log2
// - lse log2(e) (bias -10000 sqrt(d) for a padded key), and dS = P (y - D),
// each as two bf16 terms, hi = bf16(v) and lo = bf16(v - hi), packed in
// pairs: the products then see about 16 significant bits of P and dS. (One
// bf16 rounding leaves about 2^-9 relative error in each term, and dq, dk and
// dv are sums of terms of either sign, so that error would reach the
// gradients nearly undiminished.) Pairs of columns in packed f32x2 arithmetic.
template <bool kKV>
__device__ __forceinline__ void piece_pds(const uint32_t (&x)[16], const uint32_t (&y)[16], int c0, uint64_t vm,
                                          float row_c, float row_cmask, float row_d, const float* col_lse,
                                          const float* col_d, float row_bias_l2, float scale_log2, uint32_t (&pk)[8],
                                          uint32_t (&pl)[8], uint32_t (&dk)[8], uint32_t (&dl)[8]) {
  constexpr float kLog2e = 1.4426950408889634f;
  const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
#pragma unroll
  for (int c = 0; c < 16; c += 2) {
    const int col = c0 + c;
    uint64_t cc, dd;
    if (kKV) {
      // per query column: c = row bias - lse log2(e), D
      const float2 l = *reinterpret_cast<const float2*>(col_lse + col);
      const float2 d = *reinterpret_cast<const float2*>(col_d + col);
      cc = f2_fma(f2_pack(l.x, l.y), f2_pack(-kLog2e, -kLog2e), f2_pack(row_bias_l2, row_bias_l2));
      dd = f2_pack(-d.x, -d.y);
    } else {
      // per key column: the row's c, or with the masked-key bias
      cc = f2_pack(((vm >> col) & 1ull) ? row_c : row_cmask, ((vm >> (col + 1)) & 1ull) ? row_c : row_cmask);
      dd = f2_pack(-row_d, -row_d);
    }
    float t0, t1;
    f2_unpack(f2_fma(f2_pack(__uint_as_float(x[c]), __uint_as_float(x[c + 1])), sc2, cc), t0, t1);
    const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
    const uint64_t pp = f2_pack(p0, p1);
    float d0, d1;
    f2_unpack(f2_mul(pp, f2_add(f2_pack(__uint_as_float(y[c]), __uint_as_float(y[c + 1])), dd)), d0, d1);
    const uint32_t phi = pack_bf16x2(p0, p1);
    pk[c / 2] = phi;
    float r0, r1;
    f2_unpack(f2_add(pp, f2_pack(-__uint_as_float(phi << 16), -__uint_as_float(phi & 0xFFFF0000u))), r0, r1);
    pl[c / 2] = pack_bf16x2(r0, r1);
    const uint32_t hi = pack_bf16x2(d0, d1);
    dk[c / 2] = hi;
    f2_unpack(f2_add(f2_pack(d0, d1), f2_pack(-__uint_as_float(hi << 16), -__uint_as_float(hi & 0xFFFF0000u))), r0, r1);
    dl[c / 2] = pack_bf16x2(r0, r1);
  }
}

// Warps 0-7: warps w and w + 4 share the 32 stationary rows of TMEM lanes
// 32 (w & 3) .. +31 (one row per thread) and take columns 0..31 and 32..63
// of them. Per step: read S and dP and write P (dk/dv kernel) and dS over
// them as bf16 hi and lo terms; a half whose rows do not use the tile writes
// zeros. After a unit's last step: the
// epilogue, each warp its 32 of the 64 columns (dq = acc1 / sqrt(d); dv =
// acc1, dk = acc2 / sqrt(d); raw into the partial-sum slot of a split global
// unit).
template <int kD, bool kKV>
__device__ void elem_role(Smem<kD>& s, const Params& p, uint32_t tmem, const StoreMaps* smaps) {
  constexpr float kLog2e = 1.4426950408889634f;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quad = warp & 3;
  const int chalf = warp >> 2;          // columns 32 chalf .. 32 chalf + 31
  const int rowi = quad * 32 + lane;    // stationary row 0..127 (TMEM lane)
  const int half = quad >> 1;           // rows 0..63 or 64..127
  const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  const float row_bias_l2_masked = p.bias_raw * p.scale_log2;
  uint32_t g = 0, ua = 0;
  uint32_t staged = 0;  // d = 64: accumulator tiles that went out through ostage
  float row_c = 0.f, row_cmask = 0.f, row_d = 0.f, row_bias_l2 = 0.f;
  for (uint32_t ut = 0;; ++ut) {
    if (__builtin_expect(!warp_wait(smem_u32(&s.info_full[ut & 3]), (ut >> 2) & 1), 0)) { if (lane == 0) flag_timeout(p); return; }
    const Unit& ui = s.unit[ut & 3];
    if (ui.stop) break;
    const int n = ui.n;
    const int stile = half ? ui.bot : ui.top;
    const int top_tile = ui.top, bot_tile = ui.bot;  // kept: the unit slot is released before the epilogue
    const bool exists = stile >= 0;
    const int bh = ui.bh;
    const size_t row = static_cast<size_t>(bh) * p.L + static_cast<size_t>(exists ? stile : 0) * kBlock + (rowi & 63);
    if (ui.first && exists) {
      if (kKV) {
        const int b = bh / p.H;
        const bool valid = !p.seq_mask || p.seq_mask[static_cast<size_t>(b) * p.L + (row - static_cast<size_t>(bh) * p.L)] != 0;
        row_bias_l2 = valid ? 0.f : row_bias_l2_masked;
      } else {
        const float lse2 = __ldg(p.lse + row) * kLog2e;
        row_c = -lse2;
        row_cmask = row_bias_l2_masked - lse2;
        row_d = __ldg(p.dd + row);
      }
    }
    for (int e = 0; e < n; ++e, ++g) {
      const bool used = exists && ((ui.hm[e] >> half) & 1);
      const uint32_t bb = g % BGeo<kD>::kBufs;
      if (__builtin_expect(!warp_wait(smem_u32(&s.x_full[bb]), (g / BGeo<kD>::kBufs) & 1), 0)) { if (lane == 0) flag_timeout(p); return; }
      tc_fence_after();
      const int st = g % BGeo<kD>::kStages;
      if (__builtin_expect(kKV && !warp_wait(smem_u32(&s.b_full[st]), (g / BGeo<kD>::kStages) & 1), 0)) { if (lane == 0) flag_timeout(p); return; }
      // this step's S and dP columns
      const uint32_t xcol = BGeo<kD>::x_col(bb, kKV), ycol = xcol + 64;
      if (used) {
        const uint64_t vm = kKV ? ~0ull : ui.vm[e];
#pragma unroll 1
        for (int q = 2 * chalf; q < 2 * chalf + 2; ++q) {
          uint32_t x[16], y[16], pk[8], pl[8], dk[8], dl[8];
          tmem_ld16(lane_addr + xcol + 16 * q, x);
          tmem_ld16(lane_addr + ycol + 16 * q, y);
          tmem_wait_ld();
          piece_pds<kKV>(x, y, 16 * q, vm, row_c, row_cmask, row_d, s.col_lse[st], s.col_d[st], row_bias_l2,
                         p.scale_log2, pk, pl, dk, dl);
          if (kKV) {
            tmem_st8(lane_addr + xcol + hi_col(q), pk);
            tmem_st8(lane_addr + xcol + lo_col(q), pl);
          }
          tmem_st8(lane_addr + ycol + hi_col(q), dk);
          tmem_st8(lane_addr + ycol + lo_col(q), dl);
        }
      } else {
        uint32_t z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0u;
#pragma unroll
        for (int q = 2 * chalf; q < 2 * chalf + 2; ++q) {
          if (kKV) tmem_st16(lane_addr + xcol + 16 * q, z);
          tmem_st16(lane_addr + ycol + 16 * q, z);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&s.p_full[bb]));
    }
    const bool last = ui.last;
    const int split = ui.split;
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&s.info_empty[ut & 3]));
    if (!last) continue;
    // ---- epilogue: this warp's d / 2 columns of each accumulator
    if (__builtin_expect(!warp_wait(smem_u32(&s.acc_full), ua & 1), 0)) { if (lane == 0) flag_timeout(p); return; }
    tc_fence_after();
    if constexpr (kD == 64) {
      // Each accumulator goes out through ostage: every thread writes its 32
      // columns (eight 16-byte chunks of one 128-byte box row, swizzled as the
      // tensor map expects), then warp 0 stores the tile's boxes with TMA.
      const int rr = rowi & 63;
      uint8_t* srow = s.ostage + ((rowi >> 6) * 2 + chalf) * (kBlock * 128) + rr * 128;
#pragma unroll 1
      for (int a = 0; a < (kKV ? 2 : 1); ++a) {
        // acc1: dq (dq kernel) or dv; acc2: dk
        const float f = (split >= 0 || (kKV && a == 0)) ? 1.f : p.scale;
        if (warp == 0 && lane == 0) {
          bulk_wait_read_all();  // the previous tile's stores have read ostage
          mbar_arrive(smem_u32(&s.stage_free));
        }
        if (__builtin_expect(!warp_wait(smem_u32(&s.stage_free), staged & 1), 0)) { if (lane == 0) flag_timeout(p); return; }
        if (exists) {
#pragma unroll 1
          for (int c0 = 0; c0 < 32; c0 += 16) {
            uint32_t o[16];
            tmem_ld16(lane_addr + (a == 0 ? kColA1 : BGeo<kD>::kColA2) + 32 * chalf + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int cc = (c0 >> 2) + j;  // 16-byte chunk (four floats) of the box row
              *reinterpret_cast<float4*>(srow + ((cc ^ (rr & 7)) << 4)) =
                  make_float4(__uint_as_float(o[4 * j]) * f, __uint_as_float(o[4 * j + 1]) * f,
                              __uint_as_float(o[4 * j + 2]) * f, __uint_as_float(o[4 * j + 3]) * f);
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&s.tile_ready));
        if (warp == 0) {
          if (__builtin_expect(!warp_wait(smem_u32(&s.tile_ready), staged & 1), 0)) { if (lane == 0) flag_timeout(p); return; }
          if (lane == 0) {
            const CUtensorMap* map = split >= 0 ? (a == 0 ? &smaps->p1 : &smaps->p2) : (a == 0 ? &smaps->o1 : &smaps->o2);
            const uint32_t src = smem_u32(s.ostage);
            int32_t y0, y1;
            if (split >= 0) {
              y0 = (bh * p.nparts + split) * kRows;
              y1 = y0 + kBlock;
            } else {
              y0 = bh * p.L + top_tile * kBlock;
              y1 = bot_tile >= 0 ? bh * p.L + bot_tile * kBlock : -1;
            }
            tma_store_2d(map, src, 0, y0);
            tma_store_2d(map, src + kBlock * 128, 32, y0);
            if (y1 >= 0) {
              tma_store_2d(map, src + 2 * kBlock * 128, 0, y1);
              tma_store_2d(map, src + 3 * kBlock * 128, 32, y1);
            }
            bulk_commit();
          }
        }
        ++staged;
      }
    } else {
      if (exists) {
        const size_t prow = (static_cast<size_t>(bh) * p.nparts + (split >= 0 ? split : 0)) * kRows + rowi;
  #pragma unroll 1
        for (int a = 0; a < (kKV ? 2 : 1); ++a) {
          // acc1: dq (dq kernel) or dv; acc2: dk
          const float f = (split >= 0 || (kKV && a == 0)) ? 1.f : p.scale;
          float* dst = split >= 0 ? (a == 0 ? p.part1 : p.part2) + prow * kD : (a == 0 ? p.g1 : p.g2) + row * kD;
  #pragma unroll 1
          for (int c0 = (kD / 2) * chalf; c0 < (kD / 2) * (chalf + 1); c0 += 16) {
            uint32_t o[16];
            tmem_ld16(lane_addr + (a == 0 ? kColA1 : BGeo<kD>::kColA2) + c0, o);
            tmem_wait_ld();
            float4* d4 = reinterpret_cast<float4*>(dst + c0);
  #pragma unroll
            for (int c = 0; c < 4; ++c)
              d4[c] = make_float4(__uint_as_float(o[4 * c]) * f, __uint_as_float(o[4 * c + 1]) * f,
                                  __uint_as_float(o[4 * c + 2]) * f, __uint_as_float(o[4 * c + 3]) * f);
          }
        }
      }
}
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&s.acc_free));
    ++ua;
  }
}

// ------------------------------------------------------------ kernels

// kKV = false: dq. kKV = true: dk and dv. kD: head dimension; kBt: tiles per block.
template <int kD, int kBt, bool kKV>
__global__ void __launch_bounds__(kThreads, BGeo<kD>::kCtasPerSm)
bwd_kernel(const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmA2,
           const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
           const __grid_constant__ StoreMaps smaps, const __grid_constant__ Params p) {
  constexpr uint32_t kTmemCols = BGeo<kD>::tmem_cols(kKV);
  extern __shared__ uint8_t smem_raw[];
  Smem<kD>& s = *reinterpret_cast<Smem<kD>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (warp == 9) {
    tmem_alloc(smem_u32(&s.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(smem_u32(&s.info_full[i]), 1);
      mbar_init(smem_u32(&s.info_empty[i]), 1 + 2 + kElemWarps);  // TMA, two MMA threads, elementwise warps
    }
    mbar_init(smem_u32(&s.a_full), 1);
    mbar_init(smem_u32(&s.a_free), 2);  // both MMA threads read the stationary operands
    for (int i = 0; i < BGeo<kD>::kStages; ++i) {
      mbar_init(smem_u32(&s.b_full[i]), 1);
      mbar_init(smem_u32(&s.b_empty[i]), 2);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s.x_full[i]), 2);  // S and dP, one MMA thread each
      mbar_init(smem_u32(&s.p_full[i]), kElemWarps);
      mbar_init(smem_u32(&s.xy_free[0][i]), 1);
      mbar_init(smem_u32(&s.xy_free[1][i]), 1);
    }
    mbar_init(smem_u32(&s.acc_full), kKV ? 2 : 1);  // dk/dv: two accumulators, one per MMA thread
    mbar_init(smem_u32(&s.acc_free), kElemWarps);
    mbar_init(smem_u32(&s.stage_free), 1);
    mbar_init(smem_u32(&s.tile_ready), kElemWarps);
    fence_barrier_init();
  }
  // The dq kernel follows the dk/dv kernel as its programmatic dependent: it
  // reads nothing the dk/dv kernel writes, so its CTAs may take the SMs the
  // dk/dv kernel's CTAs leave (they never wait for the dk/dv grid; both read
  // D, which the row dot, launched before them in stream order, wrote).
  if (kKV) asm volatile("griddepcontrol.launch_dependents;");
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmA2);
    tma_prefetch_desc(&tmB1);
    tma_prefetch_desc(&tmB2);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  if (warp < kElemWarps) {
    elem_role<kD, kKV>(s, p, tmem, &smaps);
    // the gradient tiles' TMA stores read shared memory until they complete
    if (kD == 64 && warp == 0 && lane == 0) bulk_wait_all();
  } else if (warp == 8) {
    producer_role<kD, kKV>(s, p, &tmA1, &tmA2, &tmB1, &tmB2);
  } else if (warp == 9) {
    if (lane == 0) mma_role<kD, kKV, 0>(s, p, tmem);
  } else if (warp == 10) {
    prep_role<kD, kBt, kKV>(s, p);
  } else if (warp == 11) {
    if (lane == 0) mma_role<kD, kKV, 1>(s, p, tmem);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
  // the CTA that finishes last sets this kernel's counters back to zero
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&p.counters[1], 1) == static_cast<int>(gridDim.x) - 1) {
      p.counters[0] = 0;
      p.counters[1] = 0;
    }
  }
}

// D[row] = sum_c dout[row, c] * out[row, c]: d / 8 threads per row, 8
// columns (16 bytes of each bf16 operand) each; a CTA of 256 threads covers
// 2048 / d rows.
template <int kD>
__global__ void __launch_bounds__(256)
bwd_rowdot_kernel(const uint16_t* __restrict__ dout, const void* __restrict__ out, int out_f32, float* __restrict__ dd,
                  size_t rows) {
  constexpr int kTpr = kD / 8;
  const size_t row = static_cast<size_t>(blockIdx.x) * (256 / kTpr) + threadIdx.x / kTpr;
  const int c8 = threadIdx.x % kTpr;
  float acc = 0.f;
  if (row < rows) {
    const uint4 g = __ldg(reinterpret_cast<const uint4*>(dout + row * kD) + c8);
    float o[8];
    if (out_f32) {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(out) + row * kD) + 2 * c8;
      const float4 t0 = __ldg(src), t1 = __ldg(src + 1);
      o[0] = t0.x; o[1] = t0.y; o[2] = t0.z; o[3] = t0.w;
      o[4] = t1.x; o[5] = t1.y; o[6] = t1.z; o[7] = t1.w;
    } else {
      const uint4 t = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(out) + row * kD) + c8);
      const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        o[2 * i] = __uint_as_float(w[i] << 16);
        o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    }
    const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      acc += __uint_as_float(gw[i] << 16) * o[2 * i] + __uint_as_float(gw[i] & 0xFFFF0000u) * o[2 * i + 1];
  }
#pragma unroll
  for (int off = kTpr / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < rows && c8 == 0) dd[row] = acc;
}

// The split global units' partial sums, dst = f * sum over the ranges. Rows
// 0..63 and 64..127 of global unit g of head bh are tiles 0 and nt-1 (block
// 64: both global blocks in one unit), or the two tiles of block 0 (g = 0) or
// of block nb-1 (block 128). d / 4 threads per row, 4 columns each; grid
// (B*H*n_glob, 128 d / 1024, 3): the three gradients in one launch.
struct SumJobs {
  const float* part[3];
  float* dst[3];
  float f[3];
};

template <int kD>
__global__ void __launch_bounds__(256)
bwd_sum_kernel(const __grid_constant__ SumJobs jobs, int nsplit, int n_glob, int L, int nt) {
  constexpr int kTpr = kD / 4;
  // blockIdx.z: which gradient (dq, dv, dk)
  const float* __restrict__ part = jobs.part[blockIdx.z];
  float* __restrict__ dst = jobs.dst[blockIdx.z];
  const float f = jobs.f[blockIdx.z];
  const int bh = blockIdx.x / n_glob;
  const int g = blockIdx.x % n_glob;
  const int r = blockIdx.y * (256 / kTpr) + static_cast<int>(threadIdx.x) / kTpr;
  const int c4 = static_cast<int>(threadIdx.x) % kTpr;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const size_t base = (static_cast<size_t>(bh) * n_glob + g) * nsplit;
  for (int sidx = 0; sidx < nsplit; ++sidx) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(part + ((base + sidx) * kRows + r) * kD) + c4);
    acc.x += t.x;
    acc.y += t.y;
    acc.z += t.z;
    acc.w += t.w;
  }
  const int tile = n_glob == 1 ? (r < kBlock ? 0 : nt - 1) : (g == 0 ? 0 : nt - 2) + r / kBlock;
  const size_t row = static_cast<size_t>(bh) * L + static_cast<size_t>(tile) * kBlock + (r & (kBlock - 1));
  reinterpret_cast<float4*>(dst + row * kD)[c4] = make_float4(acc.x * f, acc.y * f, acc.z * f, acc.w * f);
}

template <int kD>
constexpr int smem_request() {
  return kD == 64 ? kSmemRequest64 : static_cast<int>(sizeof(Smem<kD>) + 1024);
}
static_assert(sizeof(Smem<64>) + 1024 <= kSmemRequest64, "shared memory request below the kernel's use");
static_assert(3 * (kSmemRequest64 + 1024) > 228 * 1024, "a third CTA per SM would wait for TMEM");
static_assert(2 * (sizeof(Smem<128>) + 2048) > 228 * 1024, "d = 128: one CTA per SM");

}  // namespace bbw

// ------------------------------------------------------------ host

namespace {

struct BwdPlan {
  int nb = 0, nt = 0, bt = 1;
  bool sparse = false;
  int nsplit = 1, n_glob = 1;
  size_t d_off = 0, partq_off = 0, partv_off = 0, partk_off = 0, bytes = 0;
};

// Blocks of 64 or 128 at d = 64 or 128; full attention wider than one unit's
// list (block 128 with r > 8) is not supported.
int bwd_plan(int B, int H, int L, int d, int block, int r, unsigned flags, BwdPlan& pl) {
  using namespace bbw;
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0 || block <= 0 || r < 1 || L % block != 0) return BB_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || (block != kBlock && block != 2 * kBlock) || r > kMaxR) return BB_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * L >= (int64_t(1) << 31)) return BB_ERR_UNSUPPORTED;
  pl.nb = L / block;
  pl.bt = block / kBlock;
  pl.nt = L / kBlock;
  pl.sparse = (flags & BB_FLAG_FORCE_SPARSE) || pl.nb > 5 + 2 * r;
  if (pl.sparse && pl.nb < 5 + r) return BB_ERR_INVALID_ARG;
  if (!pl.sparse && pl.nt > kMaxList) return BB_ERR_UNSUPPORTED;
  pl.nsplit = pl.sparse ? (pl.nt + kSplit - 1) / kSplit : 1;
  pl.n_glob = pl.sparse && pl.bt == 2 ? 2 : 1;
  auto round256 = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t bhl = static_cast<size_t>(B) * H * L;
  pl.d_off = kCounterBytes;
  size_t off = pl.d_off + round256(bhl * sizeof(float));
  if (pl.nsplit > 1) {
    const size_t part = static_cast<size_t>(B) * H * pl.n_glob * pl.nsplit * kRows * d * sizeof(float);
    pl.partq_off = off;
    pl.partv_off = off + part;
    pl.partk_off = off + 2 * part;
    off += 3 * part;
  }
  pl.bytes = off;
  return BB_OK;
}

template <int kD>
bool set_attributes_d() {
  using namespace bbw;
  const int smem = smem_request<kD>();
  for (const void* fn : {reinterpret_cast<const void*>(bwd_kernel<kD, 1, false>),
                         reinterpret_cast<const void*>(bwd_kernel<kD, 1, true>),
                         reinterpret_cast<const void*>(bwd_kernel<kD, 2, false>),
                         reinterpret_cast<const void*>(bwd_kernel<kD, 2, true>)}) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return false;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess) return false;
  }
  return true;
}

bool set_attributes(int dev) {
  static bool done[64] = {};
  if (dev < 0 || dev >= 64) return false;
  if (done[dev]) return true;
  if (!set_attributes_d<64>() || !set_attributes_d<128>()) return false;
  done[dev] = true;
  return true;
}

// The launches of one backward call: row dot, dk/dv kernel, dq kernel (its
// programmatic dependent), then the partial sums of the split global units
// (a normal launch: it waits for both attention kernels).
template <int kD, int kBt>
cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                       const bbw::StoreMaps& smq, const bbw::StoreMaps& smk, const bbw::Params& pq,
                       const bbw::Params& pk, const BwdPlan& pl, int sms, const void* dout,
                       const void* out, int out_f32, float* dd, size_t rows, float* dq, float* dk, float* dv, int L,
                       cudaStream_t stream) {
  using namespace bbw;
  const int grid = std::min(pq.total_units, BGeo<kD>::kCtasPerSm * sms);
  const size_t smem = smem_request<kD>();
  constexpr int kRowsPerCta = 256 / (kD / 4);        // partial sums: d / 4 threads per row
  constexpr int kDotRowsPerCta = 256 / (kD / 8);     // row dot: d / 8 threads per row
  bwd_rowdot_kernel<kD><<<static_cast<unsigned>((rows + kDotRowsPerCta - 1) / kDotRowsPerCta), 256, 0, stream>>>(
      static_cast<const uint16_t*>(dout), out, out_f32, dd, rows);
  const int grid_kv = std::min(pk.total_units, BGeo<kD>::kCtasPerSm * sms);
  bwd_kernel<kD, kBt, true><<<grid_kv, kThreads, smem, stream>>>(tk, tv, tq, tdo, smk, pk);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the dq kernel as the dk/dv kernel's programmatic dependent (see the kernel)
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, bwd_kernel<kD, kBt, false>, tq, tdo, tk, tv, smq, pq);
  if (e != cudaSuccess) return e;
  if (pl.nsplit > 1) {
    // a normal launch: it waits for both attention kernels
    const dim3 sg(pq.BH * pl.n_glob, kRows / kRowsPerCta, 3);
    SumJobs jobs{{pq.part1, pk.part1, pk.part2}, {dq, dv, dk}, {pq.scale, 1.0f, pq.scale}};
    bwd_sum_kernel<kD><<<sg, 256, 0, stream>>>(jobs, pl.nsplit, pl.n_glob, L, pl.nt);
  }
  return cudaGetLastError();
}

}  // namespace

extern "C" size_t bigbird_attn_bwd_workspace_size(int B, int H, int L, int d, int block, int r, unsigned flags) {
  BwdPlan pl;
  return bwd_plan(B, H, L, d, block, r, flags, pl) == BB_OK ? pl.bytes : 0;
}

extern "C" int bigbird_attn_bwd_ex(const void* q, const void* k, const void* v, const void* out, const void* dout,
                                   const float* lse, const int32_t* rand_attn, const uint8_t* seq_mask, float* dq,
                                   float* dk, float* dv, int B, int H, int L, int d, int block, int r, int out_dtype,
                                   unsigned flags, void* workspace, size_t workspace_bytes, void* stream_) {
  using namespace bbw;
  BwdPlan pl;
  const int st = bwd_plan(B, H, L, d, block, r, flags, pl);
  if (st != BB_OK) return st;
  if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv) return BB_ERR_INVALID_ARG;
  if (out_dtype != BB_OUT_BF16 && out_dtype != BB_OUT_F32) return BB_ERR_INVALID_ARG;
  if (pl.sparse && !rand_attn) return BB_ERR_INVALID_ARG;
  auto misaligned = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) != 0; };
  if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(out, 16) || misaligned(dout, 16) ||
      misaligned(lse, 16) || misaligned(dq, 16) || misaligned(dk, 16) || misaligned(dv, 16))
    return BB_ERR_UNSUPPORTED;
  if (workspace && (misaligned(workspace, 256) || workspace_bytes < pl.bytes)) return BB_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  int dev = 0, major = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BB_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return BB_ERR_CUDA;
  if (major != 10) return BB_ERR_UNSUPPORTED;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return BB_ERR_CUDA;
  uint32_t* status = status_word(dev);
  if (!status || !set_attributes(dev)) return BB_ERR_CUDA;

  const size_t rows = static_cast<size_t>(B) * H * L;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_tile_map_d(&tq, q, rows, d) || !make_tile_map_d(&tk, k, rows, d) || !make_tile_map_d(&tv, v, rows, d) ||
      !make_tile_map_d(&tdo, dout, rows, d))
    return BB_ERR_CUDA;

  void* ws = workspace;
  bool owned = false;
  if (!ws) {
    if (cudaMallocAsync(&ws, pl.bytes, stream) != cudaSuccess) return BB_ERR_CUDA;
    owned = true;
    if (cudaMemsetAsync(ws, 0, kCounterBytes, stream) != cudaSuccess) {
      cudaFreeAsync(ws, stream);
      return BB_ERR_CUDA;
    }
  }
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* dd = reinterpret_cast<float*>(wsb + pl.d_off);

  Params p{};
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.dout = static_cast<const uint16_t*>(dout);
  p.lse = lse;
  p.dd = dd;
  p.rand_attn = rand_attn;
  p.seq_mask = seq_mask;
  p.status = status;
  p.H = H;
  p.L = L;
  p.nb = pl.nb;
  p.r = r;
  p.BH = B * H;
  p.nt = pl.nt;
  p.sparse = pl.sparse ? 1 : 0;
  p.nsplit = pl.nsplit;
  p.n_glob = pl.n_glob;
  p.nparts = pl.n_glob * pl.nsplit;
  // middle units: pairs of blocks (block 64) or single blocks (block 128)
  p.n_mid_per_head = pl.sparse ? (pl.bt == 1 ? (pl.nb - 2 + 1) / 2 : pl.nb - 2) : 0;
  p.n_mid_units = p.BH * p.n_mid_per_head;
  p.total_units = p.n_mid_units + p.BH * (pl.sparse ? p.nparts : (pl.nt + 1) / 2);
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(d));
  p.bias_raw = -10000.0f * sqrtf(static_cast<float>(d));
  p.scale = 1.0f / sqrtf(static_cast<float>(d));

  Params pq = p;
  pq.g1 = dq;
  pq.part1 = pl.nsplit > 1 ? reinterpret_cast<float*>(wsb + pl.partq_off) : nullptr;
  pq.counters = reinterpret_cast<int*>(wsb);
  Params pk = p;
  pk.g1 = dv;
  pk.g2 = dk;
  pk.part1 = pl.nsplit > 1 ? reinterpret_cast<float*>(wsb + pl.partv_off) : nullptr;
  pk.part2 = pl.nsplit > 1 ? reinterpret_cast<float*>(wsb + pl.partk_off) : nullptr;
  pk.counters = reinterpret_cast<int*>(wsb) + 2;
  const int of32 = out_dtype == BB_OUT_F32 ? 1 : 0;
  // d = 64: the gradient tiles leave through TMA stores (maps over dq, dv, dk
  // and the three partial-sum arrays; unused entries repeat a valid map)
  StoreMaps smq{}, smk{};
  if (d == 64) {
    const uint64_t prow = static_cast<uint64_t>(B) * H * pl.n_glob * pl.nsplit * kRows;
    bool ok = make_f32_map(&smq.o1, dq, rows) && make_f32_map(&smk.o1, dv, rows) && make_f32_map(&smk.o2, dk, rows);
    if (ok && pl.nsplit > 1) {
      ok = make_f32_map(&smq.p1, pq.part1, prow) && make_f32_map(&smk.p1, pk.part1, prow) &&
           make_f32_map(&smk.p2, pk.part2, prow);
    } else {
      smq.p1 = smq.o1;
      smk.p1 = smk.o1;
      smk.p2 = smk.o2;
    }
    smq.o2 = smq.o1;
    smq.p2 = smq.p1;
    if (!ok) {
      if (owned) cudaFreeAsync(ws, stream);
      return BB_ERR_CUDA;
    }
  }
  cudaError_t e;
  if (d == 64)
    e = pl.bt == 1 ? launch_bwd<64, 1>(tq, tk, tv, tdo, smq, smk, pq, pk, pl, sms, dout, out, of32, dd, rows, dq, dk, dv, L, stream)
                   : launch_bwd<64, 2>(tq, tk, tv, tdo, smq, smk, pq, pk, pl, sms, dout, out, of32, dd, rows, dq, dk, dv, L, stream);
  else
    e = pl.bt == 1 ? launch_bwd<128, 1>(tq, tk, tv, tdo, smq, smk, pq, pk, pl, sms, dout, out, of32, dd, rows, dq, dk, dv, L, stream)
                   : launch_bwd<128, 2>(tq, tk, tv, tdo, smq, smk, pq, pk, pl, sms, dout, out, of32, dd, rows, dq, dk, dv, L, stream);
  if (owned) cudaFreeAsync(ws, stream);
  return e == cudaSuccess ? BB_OK : BB_ERR_CUDA;
}

extern "C" int bigbird_attn_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
                                const float* lse, const int32_t* rand_attn, const uint8_t* seq_mask, float* dq,
                                float* dk, float* dv, int B, int H, int L, int d, int block, int r, int out_dtype,
                                unsigned flags, void* stream) {
  return bigbird_attn_bwd_ex(q, k, v, out, dout, lse, rand_attn, seq_mask, dq, dk, dv, B, H, L, d, block, r, out_dtype,
                             flags, nullptr, 0, stream);
}
