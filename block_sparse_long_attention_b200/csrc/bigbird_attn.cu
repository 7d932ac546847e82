// BigBird ITC block-sparse attention forward for B200 (sm_100a).
//
// Persistent, warp-specialised kernels process "units" of 128 query rows (two
// 64-row query blocks stacked, so every tensor-core MMA has M = 128):
//
//   * global units: query blocks 0 and nb-1 (or a pair of blocks in the
//     full-attention fallback) against a contiguous range of key blocks; with
//     more than one range per head the unit writes a partial (unnormalised
//     output, running max, running sum) that the bf16 instance's grid
//     (launched behind this one) combines by log-sum-exp [TFG-BigBird, section "BigBird：从二次方注意力到线性稀疏注意力":
//     the first and last blocks attend to the whole K/V];
//   * pair units: query blocks i and i+1 (1 <= i <= nb-2) against the union of
//     their key blocks -- window, the two global blocks and their random blocks
//     rand_attn[h][i-1], rand_attn[h][i] -- with a per-block mask telling which
//     of the two 64-row halves uses the block [TFG-BigBird, same section and
//     "随机块掩码是如何生成的"; HF-Pegasus, section "三类注意力组合"]. A half that
//     does not use a block writes P = 0 for it, so the pair shares every MMA.
//
// Units are handed out dynamically (longest first): a CTA's first unit is its
// block index, later ones are tickets from a counter in the workspace; the
// CTA that finishes last sets the workspace counters back to zero.
//
// Per key block the chain is S = Q K^T (tcgen05 SS-MMA, 128x64x16 steps) ->
// softmax -> fp16 P written back over the S columns it was read from -> O +=
// P V (TS-MMA, A = P from TMEM). Two kernels run it:
//
//   * d = 64: bigbird_fwd2_kernel, two CTAs per SM, 384 threads (80
//     registers). Each row's 64 keys per block are split between two softmax
//     warps (keys 0..31 and 32..63), each with its own reference max, running
//     sum and O accumulator (O_a, O_b), combined once per unit; S is
//     double-buffered in TMEM (S0, S1, O_a, O_b: 256 columns), so S(g+1) is
//     computed while the softmax works on block g. Warps 0-7 softmax and
//     epilogue, 8 TMA (Q double-buffered, K and V on 2-deep rings released by
//     the S and P.V completions themselves), 9 TMEM and the MMAs (one
//     thread), 10 unit preparation, 11 V conversion.
//   * d = 128: bigbird_fwd_kernel, two CTAs per SM, 256 threads, one softmax
//     thread per row over the whole block, S [0,64) and O [64,192) in 256
//     TMEM columns; the next S waits for the P.V that reads P (tcgen05 only
//     orders MMAs that share an accumulator). Warps 0-3 softmax, 4 TMA, 5
//     MMA, 6 unit preparation, 7 V conversion.
//
// The prep warp schedules and prepares units (key-block list, half masks,
// key-validity bits) up to two units ahead, plus L2 prefetch, so its
// dependent global loads never stall the pipeline.
//
// Softmax: 16 columns at a time; the reference max moves only when a score
// exceeds it by more than 2^14 (rare: then the P pieces already written in
// the block are rescaled in TMEM, and O once the previous P.V has landed; the
// final O / l is exact either way). Padded keys get -10000 added to the scaled
// score. P.V runs in fp16: P is written as fp16 and each V tile is converted
// bf16 -> fp16 in shared memory (exact in the fp16 normal range), which keeps
// three more mantissa bits of P than bf16. fp16 cannot represent a magnitude
// >= 65536: the converter flags such a value (in the workspace) as it
// converts, and a second instance of the kernel, launched behind the first as
// its programmatic dependent, then recomputes the whole call with bf16 P and
// V as loaded (8 significant bits of P), so every finite bf16 V is taken.
// Without the flag the second instance only merges the global rows' ranges.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/bigbird_attn.h"
#include "bb_internal.h"
#include "sm100_ptx.cuh"

namespace bb {

constexpr int kBlock = 64;             // tokens per tile: a block of 64, or half a block of 128
constexpr int kRows = 128;             // query rows per unit (two tiles)
constexpr int kKStages = 2;            // K ring depth (blocks)
constexpr int kVStages = 2;            // V ring depth (blocks)
constexpr int kMaxList = 42;           // key tiles per unit
constexpr int kMaxR = 16;              // random blocks per row supported
constexpr int kSplitBlocks = 8;        // key tiles per global-row range
constexpr int kSplitBlocksLong = 12;   // ... at block 64, d 64 with 256 or more tiles (L >= 16384)
constexpr int kThreads = 256;
constexpr uint32_t kColO = 64;         // O: d fp32 columns
constexpr uint32_t kChunkBytes = kBlock * 64 * 2;  // 64 rows x 64 columns bf16: one TMA box, one 128-byte swizzle span

// Sizes that follow from the head dimension d (64 or 128). A row of d values
// is cut into d / 64 chunks of 64 columns; each tile is stored chunk by chunk
// (chunk c of a K or V tile at c * 8 KB, of the unit's 128 Q rows at c * 16 KB).
template <int kD>
struct Geo {
  static constexpr int kChunks = kD / 64;
  static constexpr uint32_t kTileBytes = kBlock * kD * 2;    // one 64-token tile of K or V
  static constexpr uint32_t kQChunkBytes = kRows * 64 * 2;   // one chunk of the unit's Q
  // bigbird_fwd_kernel (d = 128; d = 64 runs on bigbird_fwd2_kernel): TMEM
  // columns per CTA and CTAs per SM (TMEM and shared memory). The template
  // also describes the single-buffered d = 64 form (S 64 + O 64 in 128
  // columns, four CTAs per SM), which is no longer launched.
  static constexpr uint32_t kTmemCols = kD == 64 ? 128 : 256;
  static constexpr int kCtasPerSm = kD == 64 ? 4 : 2;
  // its S buffers: at d = 128 the second one sits in the 64 columns after O
  // (S(g+1) is computed while the softmax works on block g)
  static constexpr int kSBufs = kD == 128 ? 2 : 1;
  __host__ __device__ static constexpr uint32_t s_col(uint32_t g) { return (kSBufs == 2 && (g & 1)) ? 192u : 0u; }
};
// The reference max moves only when a score exceeds it by more than 2^14: P
// (fp16, largest finite 65504) then stays <= 2^14 with headroom, and the
// repairs of already-written P and O stay rare even for wide score ranges.
constexpr float kRescaleThreshold = 14.0f;  // log2 units
constexpr float kNegInit = -1.0e30f;

// bf16 exponent field (bits 7..14 of a 16-bit value) of 2^16: a tile whose
// largest exponent field reaches it holds a value fp16 cannot represent.
constexpr uint32_t kBigExpField = 143u << 7;

// Workspace counters (ints, in the first 256 bytes): [0] unit tickets handed
// out beyond gridDim.x, [1] CTAs finished, [2] set when a V value fp16 cannot
// represent was seen (the bf16 instance then recomputes the call).
constexpr size_t kCounterBytes = 256;
constexpr int kCtrTickets = 0, kCtrDone = 1, kCtrBigV = 2, kCtrParts = 3;

// status word bits
constexpr uint32_t kStatusBadRandAttn = 1u;
constexpr uint32_t kStatusTimeout = 2u;

__device__ uint32_t g_status;

// Everything below is counted in 64-token tiles: a block of 64 is one tile, a
// block of 128 two. A unit is 128 query rows (two tiles) against a list of key
// tiles.
struct UnitInfo {
  int32_t n;     // key tiles in the list
  int32_t bh;    // b * H + h
  int32_t qtop;  // query tile of rows 0..63
  int32_t qbot;  // query tile of rows 64..127, or -1
  int32_t split; // partial-result slot of a split global unit (global unit * nsplit + range), or -1
  int32_t stop;  // 1: no more units for this CTA (every role leaves its loop)
  int32_t kb[kMaxList];
  uint64_t vm[kMaxList];  // bit c set: key c of the block is valid
  uint8_t hm[kMaxList];   // bit 0: rows 0..63 use the block, bit 1: rows 64..127
};

struct FwdParams {
  const uint16_t* q;  // bf16 [B*H*L, 64], for L2 prefetch (loads go through the tensor maps)
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* rand_attn;
  const uint8_t* seq_mask;
  void* out;
  float* lse;      // [B*H*L] natural-log log-sum-exp of each row's scores, or null
  float* part_o;   // [BH, nparts, 128, 64]
  float* part_ml;  // [BH, nparts, 128, 2]
  uint32_t* status;
  int* counters;    // workspace counters (zero at launch; the last CTA resets them)
  int B, H, L, nb, r, BH;
  int nt;            // 64-token tiles per sequence (L / 64)
  int bt;            // tiles per block: 1 (block 64) or 2 (block 128)
  int sparse;
  int nsplit;        // key ranges per global unit (1 = write the output directly)
  int split_tiles;   // key tiles per range
  int n_glob;        // global units per range: 1 (blocks 0 and nb-1 stacked) or 2 (one per global block)
  int nparts;        // n_glob * nsplit
  int n_pair_units;  // middle units come first (they are the longer ones)
  int n_pairs;       // middle units per head
  int total_units;
  int out_f32;
  float scale_log2;  // log2(e) / sqrt(d)
  float bias_raw;    // -10000 * sqrt(d): the masked-key bias in units of q.k
};

template <int kD>
struct __align__(1024) SharedStorage {
  static constexpr int kDim = kD;
  static constexpr int kQBufs = 1;  // Q buffers (units whose Q is resident at once)
  static constexpr int kKSt = kKStages;
  static constexpr int kVSt = kVStages;
  static constexpr int kSoftmaxWarps = 4;
  static constexpr bool kFusedRelease = false;  // K/V stages released by their own barriers
  uint8_t q[kQBufs][kRows * kD * 2];           // Q of the current unit (chunks of two 64x64 tiles, SW128)
  uint8_t k[kKStages][Geo<kD>::kTileBytes];    // K tiles
  uint8_t v[kVStages][Geo<kD>::kTileBytes];    // V tiles, converted to fp16 in place
  UnitInfo unit[4];
  uint64_t info_full[4];
  uint64_t info_empty[4];
  uint64_t q_full[kQBufs];
  uint64_t q_free[kQBufs];
  uint64_t k_full[kKStages];
  uint64_t k_empty[kKStages];
  uint64_t v_full[kVStages];
  uint64_t v_conv[kVStages];
  uint64_t v_empty[kVStages];
  uint64_t s_full[2];   // S(g) is in S buffer g & 1
  uint64_t p_full[2];   // P(g) is in S buffer g & 1 (4 softmax warps)
  uint64_t pv_done[2];  // P.V(g) is complete (S buffer g & 1 reusable)
  uint64_t o_full;
  uint64_t o_free;
  uint32_t tmem_base;
  int32_t abort_flag;
};

// The d = 64 kernel with split rows (two CTAs per SM, 384 threads): each
// query row's 64 keys per block are shared by two softmax warps (keys 0..31
// and 32..63), each with its own reference max, running sum and O
// accumulator, combined once per unit; S is double-buffered in TMEM so that
// S(g+1) is computed while the softmax works on block g. TMEM columns (256):
// S/P buffers at 0 and 64 (half h of a buffer at +32h, its fp16 P over the
// first 16 of those columns), O of keys 0..31 at 128, of keys 32..63 at 192.
constexpr int kThreads2 = 384;
constexpr uint32_t kColOa = 128;
constexpr uint32_t kColOb = 192;
constexpr uint32_t kTmemCols2 = 256;

// TMA store maps of the split-row kernel's output tiles: `out` (bf16 with
// 64x64 boxes, or fp32 with 64-row x 32-column boxes) and the ranges'
// partial outputs (fp32, 64-row x 32-column boxes).
struct OutMaps {
  CUtensorMap out;
  CUtensorMap part;
};

struct __align__(1024) SharedStorage2 {
  static constexpr int kDim = 64;
  static constexpr int kQBufs = 2;  // the next unit's Q loads while this unit runs
  // Two K and two V stages, as many as S buffers: a K stage is free again once
  // the S that read it is complete (s_full), a V stage once its P.V is
  // (pv_done), and the converter's arrival joins the softmax warps' on p_full,
  // so the MMA thread waits and commits once per event.
  static constexpr int kKSt = 2;
  static constexpr int kVSt = 2;
  static constexpr int kSoftmaxWarps = 8;
  static constexpr bool kFusedRelease = true;
  uint8_t q[kQBufs][kRows * 64 * 2];
  uint8_t k[kKSt][kBlock * 64 * 2];
  uint8_t v[kVSt][kBlock * 64 * 2];  // converted to fp16 in place
  // a unit's output tile on its way out through TMA stores (128-byte swizzle):
  // bf16, two boxes of 64 rows x 64 columns; or fp32 (fp32 output, or the
  // partial result of a global-row range), four boxes of 64 rows x 32 columns
  uint8_t ostage[kRows * 64 * 4];
  UnitInfo unit[4];
  float2 mlx[2][2][kRows];  // (max, sum) per unit parity, column half, row: the halves' combine
  uint64_t info_full[4];
  uint64_t info_empty[4];
  uint64_t q_full[kQBufs];
  uint64_t q_free[kQBufs];
  uint64_t k_full[kKSt];
  uint64_t k_empty[kKSt];
  uint64_t v_full[kVSt];
  uint64_t v_conv[kVSt];
  uint64_t v_empty[kVSt];
  uint64_t s_full[2];   // S(g) is in buffer g & 1
  uint64_t p_full[2];   // all eight softmax warps have written P(g) into buffer g & 1
  uint64_t pv_done[2];  // P.V(g) is complete (buffer g & 1 reusable)
  uint64_t o_full;
  uint64_t o_free;
  uint64_t ml_ready;    // both halves' (max, sum) of the unit are in mlx
  uint64_t tile_ready;  // all eight softmax warps have written their part of ostage
  uint32_t tmem_base;
  int32_t abort_flag;
};

template <class Smem>
__device__ __forceinline__ void flag_timeout(Smem& s, const FwdParams& p) {
  atomicOr(p.status, kStatusTimeout);
  *reinterpret_cast<volatile int32_t*>(&s.abort_flag) = 1;
}

// Every lane waits (and acquires); the warp agrees on the outcome so that a
// timeout never splits the warp before a .sync.aligned instruction.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

// Decode unit u and build its key-tile list. Called by a whole warp: the
// lanes fetch the unit's random entries in parallel, lane 0 builds the list.
// Units, in order (longest first):
//   * middle units: with block 64, query blocks (i, i+1) for i = 1, 3, ...
//     (the last alone when nb - 2 is odd) against the union of their key
//     blocks, a half mask per tile telling which rows use it; with block 128,
//     query block i (its two tiles) against its own key blocks. The key
//     blocks of query block i: window i-1, i, i+1, the global blocks 0 and
//     nb-1 and rand_attn[h][i-1] [TFG-BigBird, section "BigBird：从二次方注意力到线性稀疏注意力"
//     and "随机块掩码是如何生成的"; HF-Pegasus, section "三类注意力组合"];
//   * global units: the rows of query blocks 0 and nb-1 (which attend to
//     every key) against one range of split_tiles key tiles -- both blocks in
//     one unit with block 64, one unit per block with block 128;
//   * full-attention fallback: query tiles (2j, 2j+1) against every key tile.
// kBt: tiles per block (1: block 64, 2: block 128).
template <int kBt>
__device__ void build_unit(const FwdParams& p, int u, UnitInfo& ui, int lane) {
  int n = 0;
  // one key tile, merging the half masks of a tile listed twice (set semantics)
  auto add_tile = [&](int kt, int hm) {
    for (int e = 0; e < n; ++e)
      if (ui.kb[e] == kt) {
        ui.hm[e] |= static_cast<uint8_t>(hm);
        return;
      }
    ui.kb[n] = kt;
    ui.hm[n] = static_cast<uint8_t>(hm);
    ++n;
  };
  // one key block of the pattern (its bt tiles); an entry outside [0, nb) is
  // skipped and reported
  auto add_block = [&](int kb, int hm) {
    if (kb < 0 || kb >= p.nb) {
      atomicOr(p.status, kStatusBadRandAttn);
      return;
    }
#pragma unroll
    for (int t = 0; t < kBt; ++t) add_tile(kb * kBt + t, hm);
  };
  if (u >= p.n_pair_units) {
    u -= p.n_pair_units;
    int bh, s, qtop, qbot, part;
    if (p.sparse) {
      bh = u / p.nparts;
      part = u % p.nparts;
      const int g = part / p.nsplit;  // global unit within the range
      s = part % p.nsplit;
      if (p.n_glob == 1) {
        qtop = 0;
        qbot = p.nt - 1;
      } else {
        qtop = g == 0 ? 0 : p.nt - 2;
        qbot = qtop + 1;
      }
    } else {
      const int npair = (p.nt + 1) / 2;
      bh = u / (npair * p.nsplit);
      const int rem = u % (npair * p.nsplit);
      const int pp = rem / p.nsplit;
      s = rem % p.nsplit;
      part = s;
      qtop = 2 * pp;
      qbot = 2 * pp + 1 < p.nt ? 2 * pp + 1 : -1;
    }
    if (lane == 0) {
      const int k0 = s * p.split_tiles;
      const int k1 = min(p.nt, k0 + p.split_tiles);
      for (int kt = k0; kt < k1; ++kt) add_tile(kt, 3);
      ui.bh = bh;
      ui.qtop = qtop;
      ui.qbot = qbot;
      ui.split = p.nsplit > 1 ? part : -1;
      ui.n = n;
      ui.stop = 0;
    }
  } else {
    const int bh = u / p.n_pairs;
    const int pp = u % p.n_pairs;
    const int h = bh % p.H;
    int qtop, qbot;
    if (kBt == 1) {
      const int i = 1 + 2 * pp;  // query blocks i and i + 1 (if still a middle block)
      const bool pair = i + 1 <= p.nb - 2;
      const int both = pair ? 3 : 1;
      // rand_attn rows i-1 and i are adjacent: lane t < r reads the top
      // row's entry t, lane r + t the bottom row's entry t.
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
      qtop = i;
      qbot = pair ? i + 1 : -1;
    } else {
      const int i = 1 + pp;  // query block i: tiles 2i and 2i + 1, both using every key block
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
      qtop = 2 * i;
      qbot = 2 * i + 1;
    }
    if (lane == 0) {
      ui.bh = bh;
      ui.qtop = qtop;
      ui.qbot = qbot;
      ui.split = -1;
      ui.n = n;
      ui.stop = 0;
    }
  }
}

// 64 validity bits of key tile kb of batch b (bit c: seq_mask of key c != 0).
__device__ __forceinline__ uint64_t key_valid_bits(const uint8_t* seq_mask, int L, int b, int kb) {
  const uint4* src = reinterpret_cast<const uint4*>(seq_mask + static_cast<size_t>(b) * L + static_cast<size_t>(kb) * kBlock);
  uint64_t bits = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 w = __ldg(src + i);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // one bit per byte (byte != 0), packed into 4 bits by a carry-free multiply
      const uint32_t m = __vcmpne4(ws[j], 0u) & 0x01010101u;
      bits |= static_cast<uint64_t>((m * 0x01020408u) >> 24) << (16 * i + 4 * j);
    }
  }
  return bits;
}

// ---------------------------------------------------------------- producer

// Prepare unit u's info (list, half masks, key validity bits). Whole warp.
template <int kBt>
__device__ void prep_unit(const FwdParams& p, int u, UnitInfo& ui, int lane) {
  build_unit<kBt>(p, u, ui, lane);
  __syncwarp();
  const int n = ui.n;
  const int b = ui.bh / p.H;
  // Key validity bits: lane e handles list entries e and e + 32.
  for (int e = lane; e < n; e += 32)
    ui.vm[e] = p.seq_mask ? key_valid_bits(p.seq_mask, p.L, b, ui.kb[e]) : ~0ull;
  __syncwarp();
}

// Unit preparation, up to two units ahead of the consumers: unit ut is
// claimed and prepared (into slot ut & 3) once every consumer has released
// unit ut - 2. The prep warp also schedules: a CTA's first unit is
// blockIdx.x, every later one is a ticket from a device-wide counter (units
// are numbered longest first), so CTAs that run faster take more units and
// all finish together; claiming only two ahead keeps the work a CTA holds
// when the tickets run out, and so the spread of finish times, small. Once
// the tickets run out it publishes a stop slot, which ends every role's loop.
template <class S, bool kAllTickets>
__device__ void prep_role(S& s, const FwdParams& p, int bt) {
  constexpr int kD = S::kDim;
  const int lane = threadIdx.x & 31;
  // kAllTickets: the first unit is a ticket too, so every unit is held by a
  // CTA that is running (what the bf16 instance's wait before its merge needs)
  int u = blockIdx.x;
  if (kAllTickets) {
    if (lane == 0) u = atomicAdd(&p.counters[kCtrTickets], 1);
    u = __shfl_sync(0xffffffffu, u, 0);
  }
  for (uint32_t ut = 0;; ++ut) {
    const int slot = ut & 3;
    int ok = 1;
    // at most two units ahead: unit ut - 2 released (which implies ut - 4)
    if (lane == 0) ok = ut < 2 || mbar_wait(smem_u32(&s.info_empty[(ut - 2) & 3]), ((ut - 2) >> 2) & 1);
    if (!__shfl_sync(0xffffffffu, ok, 0)) {
      if (lane == 0) flag_timeout(s, p);
      return;
    }
    UnitInfo& ui = s.unit[slot];
    if (u >= p.total_units) {
      if (lane == 0) {
        ui.stop = 1;
        mbar_arrive(smem_u32(&s.info_full[slot]));
      }
      return;
    }
    // Claim the next unit now, so the atomic's round trip overlaps this one's preparation.
    int next = 0;
    if (lane == 0) next = (kAllTickets ? 0 : static_cast<int>(gridDim.x)) + atomicAdd(&p.counters[kCtrTickets], 1);
    if (bt == 1) prep_unit<1>(p, u, ui, lane);
    else prep_unit<2>(p, u, ui, lane);
    if (lane == 0) mbar_arrive(smem_u32(&s.info_full[slot]));
    // Pull the unit's tiles into L2 now (it is up to two units ahead of the
    // TMA warp), so its TMA loads hit L2 instead of HBM: one tile per
    // lane, lanes 0..n-1 K, n..2n-1 V, 2n and 2n+1 the query blocks.
    const size_t row0 = static_cast<size_t>(ui.bh) * p.L;
    const int n = ui.n;
    for (int t = lane; t < 2 * n + 2; t += 32) {
      const uint16_t* base;
      int blk;
      if (t < n) { base = p.k; blk = ui.kb[t]; }
      else if (t < 2 * n) { base = p.v; blk = ui.kb[t - n]; }
      else { base = p.q; blk = (t == 2 * n) ? ui.qtop : ui.qbot; }
      if (blk >= 0) prefetch_l2_bulk(base + (row0 + static_cast<size_t>(blk) * kBlock) * kD, Geo<kD>::kTileBytes);
    }
    u = __shfl_sync(0xffffffffu, next, 0);
  }
}

// V blocks are converted bf16 -> fp16 in place (exact in the fp16 normal
// range) in the order the TMA warp loads them; the P.V MMA waits for v_conv.
// A value of magnitude >= 2^16 (its bf16 exponent field >= 143), which fp16
// cannot represent, sets the workspace flag that makes the bf16 instance
// recompute the call. The bf16 instance converts nothing: this warp only
// keeps the unit bookkeeping.
template <class S, bool kBf16>
__device__ void convert_role(S& s, const FwdParams& p) {
  constexpr int kD = S::kDim;
  const int lane = threadIdx.x & 31;
  uint32_t gv = 0;
  for (uint32_t ut = 0;; ++ut) {
    if (!warp_wait(smem_u32(&s.info_full[ut & 3]), (ut >> 2) & 1)) { if (lane == 0) flag_timeout(s, p); return; }
    if (s.unit[ut & 3].stop) break;
    const int n = s.unit[ut & 3].n;
    for (int e = 0; e < n && (!kBf16 || S::kFusedRelease); ++e, ++gv) {
      const int st = gv % S::kVSt;
      if (!warp_wait(smem_u32(&s.v_full[st]), (gv / S::kVSt) & 1)) { if (lane == 0) flag_timeout(s, p); return; }
      if (kBf16) {  // nothing to convert: only the arrival on p_full
        __syncwarp();
        if constexpr (S::kFusedRelease)
          if (lane == 0) mbar_arrive(smem_u32(&s.p_full[gv & 1]));
        continue;
      }
      uint4* vp = reinterpret_cast<uint4*>(s.v[st]) + lane;
      uint32_t ex = 0;  // largest bf16 exponent field seen, per 16-bit half
#pragma unroll 4
      for (int i = 0; i < static_cast<int>(Geo<kD>::kTileBytes / 16 / 32); ++i) {
        uint4 w = vp[32 * i];
        ex = __vmaxu2(ex, w.x & 0x7F807F80u);
        ex = __vmaxu2(ex, w.y & 0x7F807F80u);
        ex = __vmaxu2(ex, w.z & 0x7F807F80u);
        ex = __vmaxu2(ex, w.w & 0x7F807F80u);
        w.x = bf16x2_to_f16x2(w.x);
        w.y = bf16x2_to_f16x2(w.y);
        w.z = bf16x2_to_f16x2(w.z);
        w.w = bf16x2_to_f16x2(w.w);
        vp[32 * i] = w;
      }
      fence_proxy_async_smem();
      if (__any_sync(0xffffffffu, max(ex & 0xFFFFu, ex >> 16) >= kBigExpField) && lane == 0)
        atomicExch(&p.counters[kCtrBigV], 1);
      __syncwarp();
      if constexpr (S::kFusedRelease) {
        if (lane == 0) mbar_arrive(smem_u32(&s.p_full[gv & 1]));
      } else {
        if (lane == 0) mbar_arrive(smem_u32(&s.v_conv[st]));
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&s.info_empty[ut & 3]));
  }
}

// Two cursors walk this CTA's key blocks: the V cursor (at most as far as the
// K cursor) and the K cursor, which also loads each unit's Q when it enters
// the unit (single Q buffer: after every S of the previous unit is done).
// Loads every chunk of a tile: K and V tiles are 64 rows x d, stored chunk by
// chunk (x = 64 c of the tensor map, 8 KB apart).
template <class S>
__device__ void producer_role(S& s, const FwdParams& p, const CUtensorMap* tmQ, const CUtensorMap* tmK,
                              const CUtensorMap* tmV) {
  constexpr int kD = S::kDim;
  const int lane = threadIdx.x & 31;
  const uint64_t pol_kv = l2_policy_evict_last();
  const uint64_t pol_q = l2_policy_evict_first();
  uint32_t kut = 0, vut = 0, gk = 0, gv = 0;
  int ke = 0, ve = 0;
  bool kdone = false;
  while (!(kdone && gv == gk)) {
    // V first, so that the block the K cursor has just loaded gets its V
    // before the K cursor can block on the next unit's Q buffer.
    if (gv < gk) {
      const UnitInfo& ui = s.unit[vut & 3];
      int ok = 1;
      if (lane == 0) {
        const int st = gv % S::kVSt;
        if constexpr (S::kFusedRelease) {
          // the stage's previous tile (block gv - 2) is free once its P.V is complete
          ok = gv < 2 || mbar_wait(smem_u32(&s.pv_done[st]), ((gv >> 1) - 1) & 1);
        } else {
          ok = mbar_wait(smem_u32(&s.v_empty[st]), ((gv / S::kVSt) & 1) ^ 1);
        }
        if (ok) {
          const uint32_t vbar = smem_u32(&s.v_full[st]);
          mbar_arrive_expect_tx(vbar, Geo<kD>::kTileBytes);
#pragma unroll
          for (int c = 0; c < Geo<kD>::kChunks; ++c)
            tma_load_2d(smem_u32(s.v[st]) + c * kChunkBytes, tmV, vbar, 64 * c, ui.bh * p.L + ui.kb[ve] * kBlock,
                        pol_kv);
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) flag_timeout(s, p);
        return;
      }
      ++gv;
      if (++ve == ui.n) {
        // both cursors are done with this unit's info
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&s.info_empty[vut & 3]));
        ve = 0;
        ++vut;
      }
    }
    if (!kdone) {
      int ok = 1;
      if (ke == 0) ok = mbar_wait(smem_u32(&s.info_full[kut & 3]), (kut >> 2) & 1);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) flag_timeout(s, p);
        return;
      }
      const UnitInfo& ui = s.unit[kut & 3];
      if (ui.stop) {
        kdone = true;
        continue;
      }
      const int32_t row0 = ui.bh * p.L;
      if (lane == 0) {
        if (ke == 0) {
          const int qb = kut % S::kQBufs;
          ok = mbar_wait(smem_u32(&s.q_free[qb]), ((kut / S::kQBufs) & 1) ^ 1);
          if (ok) {
            const uint32_t qbar = smem_u32(&s.q_full[qb]);
            mbar_arrive_expect_tx(qbar, (ui.qbot >= 0 ? 2 : 1) * Geo<kD>::kTileBytes);
#pragma unroll
            for (int c = 0; c < Geo<kD>::kChunks; ++c) {
              // chunk c of the unit's 128 rows: the top tile, then the bottom one
              const uint32_t qdst = smem_u32(s.q[qb]) + c * Geo<kD>::kQChunkBytes;
              tma_load_2d(qdst, tmQ, qbar, 64 * c, row0 + ui.qtop * kBlock, pol_q);
              if (ui.qbot >= 0) tma_load_2d(qdst + kChunkBytes, tmQ, qbar, 64 * c, row0 + ui.qbot * kBlock, pol_q);
            }
          }
        }
        if (ok) {
          const int st = gk % S::kKSt;
          if constexpr (S::kFusedRelease) {
            // the stage's previous tile (block gk - 2) is free once its S is complete
            ok = gk < 2 || mbar_wait(smem_u32(&s.s_full[st]), ((gk >> 1) - 1) & 1);
          } else {
            ok = mbar_wait(smem_u32(&s.k_empty[st]), ((gk / S::kKSt) & 1) ^ 1);
          }
          if (ok) {
            const uint32_t kbar = smem_u32(&s.k_full[st]);
            mbar_arrive_expect_tx(kbar, Geo<kD>::kTileBytes);
#pragma unroll
            for (int c = 0; c < Geo<kD>::kChunks; ++c)
              tma_load_2d(smem_u32(s.k[st]) + c * kChunkBytes, tmK, kbar, 64 * c, row0 + ui.kb[ke] * kBlock, pol_kv);
          }
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) flag_timeout(s, p);
        return;
      }
      ++gk;
      if (++ke == ui.n) {
        ke = 0;
        ++kut;
      }
    }
  }
}

// ---------------------------------------------------------------- MMA issuer

// Per key block g of this CTA: S(g) = Q . K(g)^T into S buffer g % kSBufs
// once the P.V that read the P sharing those columns (kSBufs blocks back) is
// complete, then, once the softmax has written P(g), O += P(g) . V(g). With
// two buffers (d = 128) S(g) goes out before P.V(g - 1), so that it is ready
// when the softmax finishes block g - 1; the two CTAs of an SM interleave on
// the tensor pipe.
template <int kD, bool kBf16>
__device__ void mma_role(SharedStorage<kD>& s, const FwdParams& p, uint32_t tmem) {
  using Gm = Geo<kD>;
  constexpr int kB = Gm::kSBufs;
  const uint32_t idesc_s = idesc_f32acc(kRows, kBlock, true, false);    // bf16 Q . K^T, N = 64
  // fp16 P . fp16 V, or bf16 P . bf16 V in the bf16 instance; N = 64 per chunk of d
  const uint32_t idesc_o = idesc_f32acc(kRows, 64, kBf16, true);
  const uint32_t q_addr = smem_u32(s.q[0]);
  // P.V of block gb (first / last block of its unit ut)
  auto issue_pv = [&](uint32_t gb, bool first, bool last, uint32_t put) -> bool {
    const int vst = gb % kVStages;
    // the V tile: converted (fp16), or as loaded (bf16 instance)
    if (!mbar_wait(smem_u32(kBf16 ? &s.v_full[vst] : &s.v_conv[vst]), (gb / kVStages) & 1)) return false;
    if (first && !mbar_wait(smem_u32(&s.o_free), (put & 1) ^ 1)) return false;
    if (!mbar_wait(smem_u32(&s.p_full[gb % kB]), (gb / kB) & 1)) return false;
    tc_fence_after();
    const uint32_t v_addr = smem_u32(s.v[vst]);
    // O columns 64 c .. 64 c + 63 from V chunk c; K = 64 keys in steps of 16
#pragma unroll
    for (int c = 0; c < Gm::kChunks; ++c)
#pragma unroll
      for (int kk = 0; kk < kBlock / 16; ++kk)
        mma_ts(tmem + kColO + 64 * c, tmem + Gm::s_col(gb) + kk * 8,
               sdesc_sw128(v_addr + c * kChunkBytes + kk * 2048, 8192, 1024), idesc_o, (!first || kk > 0) ? 1u : 0u);
    mma_commit(smem_u32(&s.pv_done[gb % kB]));
    mma_commit(smem_u32(&s.v_empty[vst]));
    if (last) mma_commit(smem_u32(&s.o_full));
    return true;
  };
  uint32_t g = 0;
  bool pend = false, pend_first = false, pend_last = false;
  uint32_t pend_ut = 0;
  bool ok = true;
  for (uint32_t ut = 0; ok; ++ut) {
    if (!mbar_wait(smem_u32(&s.info_full[ut & 3]), (ut >> 2) & 1)) { ok = false; break; }
    if (s.unit[ut & 3].stop) break;
    if (!mbar_wait(smem_u32(&s.q_full[0]), ut & 1)) { ok = false; break; }
    const int n = s.unit[ut & 3].n;
    for (int e = 0; e < n; ++e, ++g) {
      const int kst = g % kKStages;
      if (!mbar_wait(smem_u32(&s.k_full[kst]), (g / kKStages) & 1)) { ok = false; break; }
      // S(g) overwrites the P that P.V(g - kB) reads
      if (g >= kB && !mbar_wait(smem_u32(&s.pv_done[g % kB]), ((g / kB) - 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t k_addr = smem_u32(s.k[kst]);
      // K = d in steps of 16: four steps (32 bytes apart) per 64-column chunk
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk)
        mma_ss(tmem + Gm::s_col(g), sdesc_sw128(q_addr + (kk >> 2) * Gm::kQChunkBytes + (kk & 3) * 32, 16, 1024),
               sdesc_sw128(k_addr + (kk >> 2) * kChunkBytes + (kk & 3) * 32, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
      mma_commit(smem_u32(&s.s_full[g % kB]));
      mma_commit(smem_u32(&s.k_empty[kst]));
      if (e == n - 1) mma_commit(smem_u32(&s.q_free[0]));
      if (kB == 1) {
        // one S buffer: P.V(g) right behind S(g)
        if (!issue_pv(g, e == 0, e == n - 1, ut)) { ok = false; break; }
      } else {
        // two: S(g) goes out before P.V(g - 1), so that it is ready when the
        // softmax finishes block g - 1
        if (pend && !issue_pv(g - 1, pend_first, pend_last, pend_ut)) { ok = false; break; }
        pend = true;
        pend_first = e == 0;
        pend_last = e == n - 1;
        pend_ut = ut;
      }
    }
    if (!ok) break;
    mbar_arrive(smem_u32(&s.info_empty[ut & 3]));
  }
  if (ok && pend && !issue_pv(g - 1, pend_first, pend_last, pend_ut)) ok = false;
  if (!ok) flag_timeout(s, p);
}

// ---------------------------------------------------------------- softmax + epilogue

// Per-block key validity: all keys valid (no bias), all masked (one uniform
// bias, folded into the exponent offset and the max), or mixed (per-key bias;
// only the block holding a sequence's padding boundary).
__device__ __forceinline__ bool block_mixed(uint64_t vm) { return vm != ~0ull && vm != 0ull; }
__device__ __forceinline__ float block_offset(uint64_t vm, float bias) { return vm == 0ull ? bias : 0.f; }

// Add the per-key bias of a mixed block to 16 raw scores (in place; vm16 bit
// c: key c valid) and return their max (q.k units, without the block offset).
__device__ __forceinline__ float piece16_prepare(uint32_t (&r)[16], bool mixed, uint32_t vm16, float bias) {
  if (mixed) {
#pragma unroll
    for (int c = 0; c < 16; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) + (((vm16 >> c) & 1u) ? 0.f : bias));
  }
  float a = fmax3(__uint_as_float(r[0]), __uint_as_float(r[1]), __uint_as_float(r[2]));
  float b = fmax3(__uint_as_float(r[3]), __uint_as_float(r[4]), __uint_as_float(r[5]));
  a = fmax3(a, __uint_as_float(r[6]), __uint_as_float(r[7]));
  b = fmax3(b, __uint_as_float(r[8]), __uint_as_float(r[9]));
  a = fmax3(a, __uint_as_float(r[10]), __uint_as_float(r[11]));
  b = fmax3(b, __uint_as_float(r[12]), __uint_as_float(r[13]));
  return fmax3(a, b, fmaxf(__uint_as_float(r[14]), __uint_as_float(r[15])));
}

// p = exp2(r * scale + off) for 16 scores, packed in pairs into pk (fp16, or
// bf16 in the bf16 instance); the sum accumulates into two packed pairs.
template <bool kBf16>
__device__ __forceinline__ void piece16_exp(const uint32_t (&r)[16], uint64_t scale2, uint64_t off2, uint32_t (&pk)[8],
                                            uint64_t& acc0, uint64_t& acc1) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float t0, t1;
    f2_unpack(f2_fma(f2_pack(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1])), scale2, off2), t0, t1);
    const float e0 = ex2_approx(t0);
    const float e1 = ex2_approx(t1);
    if (c & 1) acc1 = f2_add(acc1, f2_pack(e0, e1));
    else acc0 = f2_add(acc0, f2_pack(e0, e1));
    pk[c] = kBf16 ? pack_bf16x2(e0, e1) : pack_f16x2(e0, e1);
  }
}

// Rare path: the reference max grew inside a block after `npieces` 16-key
// pieces of P were already written (fp16, or bf16 when kBf16; 8 columns
// each): scale them by f.
template <bool kBf16>
__device__ __noinline__ void rescale_p(uint32_t s_addr, int npieces, float f) {
  tmem_wait_st();
  for (int i = 0; i < npieces; ++i) {
    uint32_t t[8];
    tmem_ld8(s_addr + 8 * i, t);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (kBf16) {
        t[j] = pack_bf16x2(__uint_as_float(t[j] << 16) * f, __uint_as_float(t[j] & 0xFFFF0000u) * f);
      } else {
        const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&t[j]));
        t[j] = pack_f16x2(v.x * f, v.y * f);
      }
    }
    tmem_st8(s_addr + 8 * i, t);
  }
  tmem_wait_st();
}

// O (64 fp32 columns of this thread's row) *= f, in 16-column pieces.
template <int kD>
__device__ __forceinline__ void rescale_o(uint32_t taddr, float f) {
#pragma unroll 1
  for (int c0 = 0; c0 < kD; c0 += 16) {
    uint32_t t[16];
    tmem_ld16(taddr + c0, t);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i) t[i] = __float_as_uint(__uint_as_float(t[i]) * f);
    tmem_st16(taddr + c0, t);
  }
  tmem_wait_st();
}

// Store 16 columns [c0, c0+16) of one output row: o * inv as bf16 or fp32.
template <int kD>
__device__ __forceinline__ void store16(const FwdParams& p, size_t row, int c0, const uint32_t (&o)[16], float inv) {
  if (p.out_f32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * kD + c0);
#pragma unroll
    for (int c = 0; c < 4; ++c)
      dst[c] = make_float4(__uint_as_float(o[4 * c]) * inv, __uint_as_float(o[4 * c + 1]) * inv,
                           __uint_as_float(o[4 * c + 2]) * inv, __uint_as_float(o[4 * c + 3]) * inv);
  } else {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + row * kD + c0);
#pragma unroll
    for (int c = 0; c < 2; ++c)
      dst[c] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * c]) * inv, __uint_as_float(o[8 * c + 1]) * inv),
                          pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv),
                          pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv),
                          pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv));
  }
}

// Warps 0..3, one query row per thread (TMEM lane = row of the unit). Per key
// block: one pass over its 64 S columns, 16 at a time -- max, a change of the
// reference max when a score exceeds it by more than 2^14 (rare; the P pieces
// already written and, after the previous P.V has landed, O are rescaled),
// exponentials, fp16 P written over the S columns already read (16 keys = 8
// columns per piece) -- then the block goes to the MMA.
template <int kD, bool kBf16>
__device__ void softmax_role(SharedStorage<kD>& s, const FwdParams& p, uint32_t tmem) {
  const int tid = threadIdx.x;  // 0..127 == TMEM lane
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int half = warp >> 1;   // 0: rows 0..63, 1: rows 64..127
  const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  constexpr int kB = Geo<kD>::kSBufs;
  const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
  uint32_t g = 0;
  for (uint32_t ut = 0;; ++ut) {
    if (!warp_wait(smem_u32(&s.info_full[ut & 3]), (ut >> 2) & 1)) { flag_timeout(s, p); return; }
    const UnitInfo& ui = s.unit[ut & 3];
    if (ui.stop) break;
    const int n = ui.n;
    const int bh = ui.bh;
    const int qblk = half ? ui.qbot : ui.qtop;
    const int split = ui.split;
    const bool exists = qblk >= 0;
    float m_ref = kNegInit;
    float l_run = 0.f;
    for (int e = 0; e < n; ++e, ++g) {
      const bool used = exists && ((ui.hm[e] >> half) & 1);
      if (!warp_wait(smem_u32(&s.s_full[g % kB]), (g / kB) & 1)) { flag_timeout(s, p); return; }
      tc_fence_after();
      const uint32_t s_addr = lane_addr + Geo<kD>::s_col(g);
      if (used) {
        const uint64_t vm = ui.vm[e];
        const bool mixed = block_mixed(vm);
        const float off = block_offset(vm, p.bias_raw);
        const float off_s = off * p.scale_log2;
        float o_factor = 1.f;  // rescale owed to O (the P.V of the earlier blocks)
        uint64_t acc0 = 0ull, acc1 = 0ull;
        uint32_t r0[16], r1[16];
        // One pass over the block's 64 columns, 16 at a time with the next
        // piece's TMEM read in flight: max, a change of the reference max when
        // it grows by more than 2^14, exponentials, and fp16 P written over S
        // columns already read (piece q -> columns 8q..8q+7).
        tmem_ld16(s_addr, r0);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t (&cur)[16] = (q & 1) ? r1 : r0;
          uint32_t (&nxt)[16] = (q & 1) ? r0 : r1;
          if (q < 3) tmem_ld16(s_addr + 16 * (q + 1), nxt);
          const float mx = fmaf(piece16_prepare(cur, mixed, static_cast<uint32_t>(vm >> (16 * q)) & 0xFFFFu,
                                                p.bias_raw),
                                p.scale_log2, off_s);
          const bool need = mx > m_ref + kRescaleThreshold;
          if (__any_sync(0xffffffffu, need)) {
            float f = 1.f;
            if (need) {
              f = ex2_approx(m_ref - mx);
              m_ref = mx;
            }
            l_run *= f;
            const uint64_t f2 = f2_pack(f, f);
            acc0 = f2_fma(acc0, f2, 0ull);
            acc1 = f2_fma(acc1, f2, 0ull);
            o_factor *= f;
            if (q > 0 && __any_sync(0xffffffffu, f != 1.f)) rescale_p<kBf16>(s_addr, q, f);
          }
          const float o = off_s - m_ref;
          uint32_t pk[8];
          piece16_exp<kBf16>(cur, scale2, f2_pack(o, o), pk, acc0, acc1);
          if (q < 3) tmem_wait_ld();
          tmem_st8(s_addr + 8 * q, pk);
        }
        float a0, a1, b0, b1;
        f2_unpack(acc0, a0, a1);
        f2_unpack(acc1, b0, b1);
        l_run += (a0 + a1) + (b0 + b1);
        // O holds the P.V of the earlier blocks (none yet for e == 0: the
        // first P.V of the unit overwrites O); rescale it once that P.V is done.
        if (e > 0 && __any_sync(0xffffffffu, o_factor != 1.f)) {
          if (!warp_wait(smem_u32(&s.pv_done[(g - 1) % kB]), ((g - 1) / kB) & 1)) { flag_timeout(s, p); return; }
          tc_fence_after();
          rescale_o<kD>(lane_addr + kColO, o_factor);
        }
      } else {
        // No row of this warp uses the block: P = 0.
        uint32_t z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0u;
        tmem_st16(s_addr, z);
        tmem_st16(s_addr + 16, z);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&s.p_full[g % kB]));
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&s.info_empty[ut & 3]));

    // ---- epilogue: O in 16-column pieces, freed after the last piece
    if (!warp_wait(smem_u32(&s.o_full), ut & 1)) { flag_timeout(s, p); return; }
    tc_fence_after();
    if (split >= 0) {
      const size_t base = (static_cast<size_t>(bh) * p.nparts + split) * kRows + tid;
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += 16) {
        uint32_t o[16];
        tmem_ld16(lane_addr + kColO + c0, o);
        tmem_wait_ld();
        float4* dst = reinterpret_cast<float4*>(p.part_o + base * kD + c0);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          dst[c] = make_float4(__uint_as_float(o[4 * c]), __uint_as_float(o[4 * c + 1]), __uint_as_float(o[4 * c + 2]),
                               __uint_as_float(o[4 * c + 3]));
      }
      reinterpret_cast<float2*>(p.part_ml)[base] = make_float2(m_ref, l_run);
      if (kBf16) {
        // the bf16 instance merges inside its own grid: count this warp's rows of the partial as written
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          atomicAdd(&p.counters[kCtrParts], 1);
        }
      }
    } else if (exists) {
      const float inv = 1.f / l_run;
      const size_t row = static_cast<size_t>(bh) * p.L + static_cast<size_t>(qblk) * kBlock + (tid & 63);
      // log sum_k exp(s_k) = ln 2 * (m_ref + log2 l), the scores in log2 units being s * log2(e).
      if (p.lse) p.lse[row] = (m_ref + log2f(l_run)) * 0.69314718055994531f;
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += 16) {
        uint32_t o[16];
        tmem_ld16(lane_addr + kColO + c0, o);
        tmem_wait_ld();
        store16<kD>(p, row, c0, o, inv);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&s.o_free));
  }
}

// ---------------------------------------------------------------- split-row kernel (d = 64)

// Per key block g of this CTA: S(g) = Q . K(g)^T into S buffer g & 1 once
// P.V(g - 2), which read the P held there, has completed; then P.V(g - 1),
// once all eight softmax warps have written P(g - 1) and the converter has
// converted V(g - 1) (both arrive on p_full): keys 0..31 into O_a,
// keys 32..63 into O_b. S(g) goes out before P.V(g - 1), so that it is ready
// when the softmax finishes block g - 1.
template <bool kBf16>
__device__ void mma2_role(SharedStorage2& s, const FwdParams& p, uint32_t tmem) {
  constexpr int kK = SharedStorage2::kKSt;
  constexpr int kV = SharedStorage2::kVSt;
  const uint32_t idesc_s = idesc_f32acc(kRows, kBlock, true, false);  // bf16 Q . K^T, N = 64
  const uint32_t idesc_o = idesc_f32acc(kRows, 64, kBf16, true);      // fp16 (or bf16) P . V, N = 64
  // P.V of block gb: first / last block of its unit, the unit's index
  auto issue_pv = [&](uint32_t gb, bool first, bool last, uint32_t put) -> bool {
    const int vst = gb % kV;
    if (first && !mbar_wait(smem_u32(&s.o_free), (put & 1) ^ 1)) return false;
    if (!mbar_wait(smem_u32(&s.p_full[gb & 1]), (gb >> 1) & 1)) return false;
    tc_fence_after();
    const uint32_t v_addr = smem_u32(s.v[vst]);
    const uint32_t pb = tmem + 64 * (gb & 1);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int kk = 0; kk < 2; ++kk)  // keys 32h + 16kk .. +15: P columns 32h + 8kk, V rows 2048 bytes apart
        mma_ts(tmem + kColOa + 64 * h, pb + 32 * h + 8 * kk, sdesc_sw128(v_addr + (2 * h + kk) * 2048, 8192, 1024),
               idesc_o, (!first || kk > 0) ? 1u : 0u);
    mma_commit(smem_u32(&s.pv_done[gb & 1]));
    if (last) mma_commit(smem_u32(&s.o_full));
    return true;
  };
  uint32_t g = 0;
  bool pend = false, pend_first = false, pend_last = false;
  uint32_t pend_ut = 0;
  bool ok = true;
  for (uint32_t ut = 0; ok; ++ut) {
    if (!mbar_wait(smem_u32(&s.info_full[ut & 3]), (ut >> 2) & 1)) { ok = false; break; }
    if (s.unit[ut & 3].stop) break;
    const int qb = ut & 1;
    if (!mbar_wait(smem_u32(&s.q_full[qb]), (ut >> 1) & 1)) { ok = false; break; }
    const uint32_t q_addr = smem_u32(s.q[qb]);
    const int n = s.unit[ut & 3].n;
    for (int e = 0; e < n; ++e, ++g) {
      const int kst = g % kK;
      if (!mbar_wait(smem_u32(&s.k_full[kst]), (g / kK) & 1)) { ok = false; break; }
      if (g >= 2 && !mbar_wait(smem_u32(&s.pv_done[g & 1]), ((g >> 1) - 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t k_addr = smem_u32(s.k[kst]);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem + 64 * (g & 1), sdesc_sw128(q_addr + kk * 32, 16, 1024), sdesc_sw128(k_addr + kk * 32, 16, 1024),
               idesc_s, kk > 0 ? 1u : 0u);
      mma_commit(smem_u32(&s.s_full[g & 1]));
      if (e == n - 1) mma_commit(smem_u32(&s.q_free[qb]));
      if (pend && !issue_pv(g - 1, pend_first, pend_last, pend_ut)) { ok = false; break; }
      pend = true;
      pend_first = e == 0;
      pend_last = e == n - 1;
      pend_ut = ut;
    }
    if (!ok) break;
    mbar_arrive(smem_u32(&s.info_empty[ut & 3]));
  }
  if (ok && pend && !issue_pv(g - 1, pend_first, pend_last, pend_ut)) ok = false;
  if (!ok) flag_timeout(s, p);
}

// Warps 0..7: warp w takes rows 32 (w % 4) .. + 31 (its TMEM lanes) and keys
// 32 (w / 4) .. + 31 of every block: one pass over those 32 S columns, 16 at a
// time (max, a change of its own reference max when a score exceeds it by
// more than 2^14, exponentials, fp16 P written over the columns already
// read), then the block goes to the MMA. At the end of a unit the two halves
// of a row exchange (max, sum) through shared memory; each writes 32 of the
// row's output columns, O_a and O_b scaled to the common max.
template <bool kBf16>
__device__ void softmax2_role(SharedStorage2& s, const FwdParams& p, uint32_t tmem, const OutMaps* tmO) {
  const int wid = threadIdx.x >> 5;  // 0..7
  const int h = wid >> 2;            // key half of each block
  const int row = threadIdx.x & 127; // TMEM lane == row of the unit
  const int lane = threadIdx.x & 31;
  const int rhalf = (wid & 3) >> 1;  // 0: rows 0..63, 1: rows 64..127
  const uint32_t lane_addr = tmem + (static_cast<uint32_t>((wid & 3) * 32) << 16);
  const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
  uint32_t g = 0;
  uint32_t staged = 0;  // units whose output tile went out through ostage
  for (uint32_t ut = 0;; ++ut) {
    if (__builtin_expect(!warp_wait(smem_u32(&s.info_full[ut & 3]), (ut >> 2) & 1), 0)) { flag_timeout(s, p); return; }
    const UnitInfo& ui = s.unit[ut & 3];
    if (ui.stop) break;
    const int n = ui.n;
    const int bh = ui.bh;
    const int qtop = ui.qtop;  // kept: the unit slot is released before the epilogue
    const int qbot = ui.qbot;
    const int qblk = rhalf ? qbot : qtop;
    const int split = ui.split;
    const bool exists = qblk >= 0;
    float m_ref = kNegInit;
    float l_run = 0.f;
    for (int e = 0; e < n; ++e, ++g) {
      const bool used = exists && ((ui.hm[e] >> rhalf) & 1);
      if (__builtin_expect(!warp_wait(smem_u32(&s.s_full[g & 1]), (g >> 1) & 1), 0)) { flag_timeout(s, p); return; }
      tc_fence_after();
      const uint32_t s_addr = lane_addr + 64 * (g & 1) + 32 * h;
      if (used) {
        const uint32_t vm = static_cast<uint32_t>(ui.vm[e] >> (32 * h));
        const bool mixed = vm != 0xFFFFFFFFu && vm != 0u;
        const float off_s = (vm == 0u ? p.bias_raw : 0.f) * p.scale_log2;
        uint32_t r0[16], r1[16];
        tmem_ld16(s_addr, r0);
        tmem_ld16(s_addr + 16, r1);
        tmem_wait_ld();
        // one reference-max decision for the 32 scores: it moves only when one
        // exceeds it by more than 2^14 (rare after a unit's first block)
        const float mx = fmaf(fmaxf(piece16_prepare(r0, mixed, vm & 0xFFFFu, p.bias_raw),
                                    piece16_prepare(r1, mixed, vm >> 16, p.bias_raw)),
                              p.scale_log2, off_s);
        const bool need = mx > m_ref + kRescaleThreshold;
        float o_factor = 1.f;  // rescale owed to O (the P.V of the earlier blocks)
        if (__builtin_expect(__any_sync(0xffffffffu, need), 0)) {
          if (need) {
            o_factor = ex2_approx(m_ref - mx);
            m_ref = mx;
          }
          l_run *= o_factor;
        }
        const float o = off_s - m_ref;
        uint64_t acc0 = 0ull, acc1 = 0ull;
        uint32_t pk0[8], pk1[8];
        piece16_exp<kBf16>(r0, scale2, f2_pack(o, o), pk0, acc0, acc1);
        piece16_exp<kBf16>(r1, scale2, f2_pack(o, o), pk1, acc0, acc1);
        tmem_st8(s_addr, pk0);
        tmem_st8(s_addr + 8, pk1);
        float a0, a1, b0, b1;
        f2_unpack(acc0, a0, a1);
        f2_unpack(acc1, b0, b1);
        l_run += (a0 + a1) + (b0 + b1);
        // this half's O holds the P.V of the earlier blocks (none yet for e == 0);
        // rescale it once that P.V is done
        if (__builtin_expect(e > 0 && __any_sync(0xffffffffu, o_factor != 1.f), 0)) {
          if (__builtin_expect(!warp_wait(smem_u32(&s.pv_done[(g - 1) & 1]), ((g - 1) >> 1) & 1), 0)) { flag_timeout(s, p); return; }
          tc_fence_after();
          rescale_o<64>(lane_addr + kColOa + 64 * h, o_factor);
        }
      } else {
        // No row of this warp uses the block: P = 0.
        uint32_t z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0u;
        tmem_st16(s_addr, z);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&s.p_full[g & 1]));
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&s.info_empty[ut & 3]));

    // ---- epilogue: combine the halves, each writes 32 columns of its row
    if (__builtin_expect(!warp_wait(smem_u32(&s.o_full), ut & 1), 0)) { flag_timeout(s, p); return; }
    tc_fence_after();
    // the previous tile's TMA store has read ostage before anyone writes it again
    if (wid == 0 && lane == 0) bulk_wait_read_all();
    s.mlx[ut & 1][h][row] = make_float2(m_ref, l_run);
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&s.ml_ready));
    if (__builtin_expect(!warp_wait(smem_u32(&s.ml_ready), ut & 1), 0)) { flag_timeout(s, p); return; }
    const float2 A = s.mlx[ut & 1][0][row];
    const float2 B = s.mlx[ut & 1][1][row];
    const float m = fmaxf(A.x, B.x);
    const float fa = ex2_approx(A.x - m);
    const float fb = ex2_approx(B.x - m);
    const float l = A.y * fa + B.y * fb;
    const int c_base = 32 * h;
    if (split >= 0 || p.out_f32) {
      // fp32 (a range's partial result, or fp32 output): each thread puts its
      // 32 columns (eight 16-byte chunks, one 128-byte box row) into ostage,
      // swizzled as the tensor map expects; warp 0 then stores the tile's
      // boxes with TMA.
      const bool has = split >= 0 || exists;
      if (has) {
        const float inv = split >= 0 ? 1.f : 1.f / l;  // a partial stays unnormalised
        if (split >= 0) {
          if (h == 0) {
            const size_t base = (static_cast<size_t>(bh) * p.nparts + split) * kRows + row;
            reinterpret_cast<float2*>(p.part_ml)[base] = make_float2(m, l);
          }
        } else if (h == 0 && p.lse) {
          const size_t orow = static_cast<size_t>(bh) * p.L + static_cast<size_t>(qblk) * kBlock + (row & 63);
          // log sum_k exp(s_k) = ln 2 * (m + log2 l), the scores in log2 units being s * log2(e).
          p.lse[orow] = (m + log2f(l)) * 0.69314718055994531f;
        }
        const int rr = row & 63;
        uint8_t* srow = s.ostage + ((row >> 6) * 2 + h) * (kBlock * 128) + rr * 128;
#pragma unroll 1
        for (int c0 = 0; c0 < 32; c0 += 16) {
          uint32_t oa[16], ob[16];
          tmem_ld16(lane_addr + kColOa + c_base + c0, oa);
          tmem_ld16(lane_addr + kColOb + c_base + c0, ob);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int cc = (c0 >> 2) + j;  // 16-byte chunk (four floats) of the box row
            *reinterpret_cast<float4*>(srow + ((cc ^ (rr & 7)) << 4)) =
                make_float4((__uint_as_float(oa[4 * j]) * fa + __uint_as_float(ob[4 * j]) * fb) * inv,
                            (__uint_as_float(oa[4 * j + 1]) * fa + __uint_as_float(ob[4 * j + 1]) * fb) * inv,
                            (__uint_as_float(oa[4 * j + 2]) * fa + __uint_as_float(ob[4 * j + 2]) * fb) * inv,
                            (__uint_as_float(oa[4 * j + 3]) * fa + __uint_as_float(ob[4 * j + 3]) * fb) * inv);
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&s.tile_ready));
      if (wid == 0) {
        if (__builtin_expect(!warp_wait(smem_u32(&s.tile_ready), staged & 1), 0)) { flag_timeout(s, p); return; }
        if (lane == 0) {
          const CUtensorMap* map = split >= 0 ? &tmO->part : &tmO->out;
          int32_t y0, y1;
          if (split >= 0) {
            y0 = (bh * p.nparts + split) * kRows;
            y1 = y0 + kBlock;
          } else {
            y0 = bh * p.L + qtop * kBlock;
            y1 = qbot >= 0 ? bh * p.L + qbot * kBlock : -1;
          }
          const uint32_t src = smem_u32(s.ostage);
          tma_store_2d(map, src, 0, y0);
          tma_store_2d(map, src + kBlock * 128, 32, y0);
          if (y1 >= 0) {
            tma_store_2d(map, src + 2 * kBlock * 128, 0, y1);
            tma_store_2d(map, src + 3 * kBlock * 128, 32, y1);
          }
          bulk_commit();
          if (kBf16 && split >= 0) {
            // the bf16 instance merges inside its own grid: count the range's
            // partial as written once the stores have completed (eight
            // softmax warps' rows; the (max, sum) pairs were written before
            // tile_ready)
            bulk_wait_all();
            __threadfence();
            atomicAdd(&p.counters[kCtrParts], SharedStorage2::kSoftmaxWarps);
          }
        }
      }
      ++staged;
    } else {
      // bf16 output: each thread puts its 32 columns (four 16-byte chunks of
      // its 128-byte row) into ostage, swizzled as the tensor map expects;
      // warp 0 then stores the tile's one or two 64-row boxes with TMA.
      if (exists) {
        const float inv = 1.f / l;
        if (h == 0 && p.lse) {
          const size_t orow = static_cast<size_t>(bh) * p.L + static_cast<size_t>(qblk) * kBlock + (row & 63);
          p.lse[orow] = (m + log2f(l)) * 0.69314718055994531f;
        }
        const int rr = row & 63;
        uint8_t* srow = s.ostage + (row >> 6) * (kBlock * 128) + rr * 128;
#pragma unroll 1
        for (int c0 = 0; c0 < 32; c0 += 16) {
          uint32_t oa[16], ob[16];
          tmem_ld16(lane_addr + kColOa + c_base + c0, oa);
          tmem_ld16(lane_addr + kColOb + c_base + c0, ob);
          tmem_wait_ld();
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            w[i] = pack_bf16x2((__uint_as_float(oa[2 * i]) * fa + __uint_as_float(ob[2 * i]) * fb) * inv,
                               (__uint_as_float(oa[2 * i + 1]) * fa + __uint_as_float(ob[2 * i + 1]) * fb) * inv);
          const int cc = (c_base + c0) >> 3;  // 16-byte chunk of the row
          *reinterpret_cast<uint4*>(srow + ((cc ^ (rr & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(srow + (((cc + 1) ^ (rr & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&s.tile_ready));
      if (wid == 0) {
        if (__builtin_expect(!warp_wait(smem_u32(&s.tile_ready), staged & 1), 0)) { flag_timeout(s, p); return; }
        if (lane == 0) {
          const int32_t row0 = bh * p.L;
          tma_store_2d(&tmO->out, smem_u32(s.ostage), 0, row0 + qtop * kBlock);
          if (qbot >= 0) tma_store_2d(&tmO->out, smem_u32(s.ostage) + kBlock * 128, 0, row0 + qbot * kBlock);
          bulk_commit();
        }
      }
      ++staged;
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&s.o_free));
  }
}

// Combine the partial results of the key ranges of the global rows by
// log-sum-exp (log2 units) and write those rows' output and lse. Called by
// every thread of a CTA; the grid's CTAs deal the rows out among themselves,
// d / 4 threads per row (4 columns each), which take the row's ranges in
// order, eight at a time with their loads in flight together. The result does
// not depend on which CTA merges a row.
template <int kD, int kNT>
__device__ void merge_ranges(const FwdParams& p, int cta, int ncta) {
  constexpr int kTpr = kD / 4;
  constexpr int kRowsPerPass = kNT / kTpr;
  constexpr int kBatch = 8;
  const int c4 = static_cast<int>(threadIdx.x) % kTpr;
  const int total = p.BH * p.n_glob * kRows;
  const float2* ml = reinterpret_cast<const float2*>(p.part_ml);
#pragma unroll 1
  for (int R = cta * kRowsPerPass + static_cast<int>(threadIdx.x) / kTpr; R < total; R += ncta * kRowsPerPass) {
    const int unit = R / kRows;  // b * H * n_glob + global unit
    const int row = R % kRows;
    const size_t base = static_cast<size_t>(unit) * p.nsplit * kRows + row;
    float m = kNegInit, l = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
    for (int s0 = 0; s0 < p.nsplit; s0 += kBatch) {
      float2 e[kBatch];
      float4 o[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        if (s0 + i < p.nsplit) {
          const size_t idx = base + static_cast<size_t>(s0 + i) * kRows;
          e[i] = __ldcg(ml + idx);
          o[i] = __ldcg(reinterpret_cast<const float4*>(p.part_o + idx * kD) + c4);
        } else {
          e[i] = make_float2(kNegInit, 0.f);
          o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      float mb = m;
#pragma unroll
      for (int i = 0; i < kBatch; ++i) mb = fmaxf(mb, e[i].x);
      const float f = ex2_approx(m - mb);
      l *= f;
      acc.x *= f;
      acc.y *= f;
      acc.z *= f;
      acc.w *= f;
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const float w = ex2_approx(e[i].x - mb);
        l += w * e[i].y;
        acc.x += w * o[i].x;
        acc.y += w * o[i].y;
        acc.z += w * o[i].z;
        acc.w += w * o[i].w;
      }
      m = mb;
    }
    const int g = unit % p.n_glob;
    const int bh = unit / p.n_glob;
    const float inv = 1.f / l;
    // rows 0..63 and 64..127 of the unit: tiles 0 and nt-1 (block 64: blocks 0
    // and nb-1 stacked), or the two tiles of block 0 (g = 0) or of block nb-1
    const int qtile = p.n_glob == 1 ? (row < kBlock ? 0 : p.nt - 1) : (g == 0 ? 0 : p.nt - 2) + row / kBlock;
    const size_t orow = static_cast<size_t>(bh) * p.L + static_cast<size_t>(qtile) * kBlock + (row & (kBlock - 1));
    if (p.lse && c4 == 0) p.lse[orow] = (m + log2f(l)) * 0.69314718055994531f;
    if (p.out_f32) {
      reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow * kD)[c4] =
          make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    } else {
      reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.out) + orow * kD)[c4] =
          make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
    }
  }
}

// kBf16 = false: the fp16 instance (every call). kBf16 = true: the bf16
// instance, launched behind it as its programmatic dependent, which merges the
// fp16 instance's global-row ranges, or, when the fp16 instance saw a V value
// fp16 cannot represent, does the whole call again and then merges its own.
// kD: the head dimension (64 or 128).
template <int kD, bool kBf16>
__global__ void __launch_bounds__(kThreads, Geo<kD>::kCtasPerSm)
bigbird_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  static_assert(kD == 128, "d = 64 runs on bigbird_fwd2_kernel");
  extern __shared__ uint8_t smem_raw[];
  SharedStorage<kD>& s =
      *reinterpret_cast<SharedStorage<kD>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (kBf16) {
    // Wait until the fp16 instance has completed (its writes visible), then
    // do the call again only if it set the flag.
    asm volatile("griddepcontrol.launch_dependents;");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // Merge the fp16 instance's ranges at once (the flag's load overlaps the
    // merge); when the flag is set the call is redone and merged again.
    int big_v = 0;
    if (threadIdx.x == 0) big_v = *reinterpret_cast<volatile int*>(&p.counters[kCtrBigV]);
    if (p.nsplit > 1) merge_ranges<kD, kThreads>(p, blockIdx.x, gridDim.x);
    if (threadIdx.x == 0) s.abort_flag = big_v;
    __syncthreads();
    if (s.abort_flag == 0) return;
    __syncthreads();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(&s.tmem_base), Geo<kD>::kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(smem_u32(&s.info_full[i]), 1);
      mbar_init(smem_u32(&s.info_empty[i]), 1 + 1 + 4 + 1);  // TMA, MMA, 4 softmax warps, converter
    }
    mbar_init(smem_u32(&s.q_full[0]), 1);
    mbar_init(smem_u32(&s.q_free[0]), 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(smem_u32(&s.k_full[i]), 1);
      mbar_init(smem_u32(&s.k_empty[i]), 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(smem_u32(&s.v_full[i]), 1);
      mbar_init(smem_u32(&s.v_conv[i]), 1);
      mbar_init(smem_u32(&s.v_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s.s_full[i]), 1);
      mbar_init(smem_u32(&s.p_full[i]), 4);
      mbar_init(smem_u32(&s.pv_done[i]), 1);
    }
    mbar_init(smem_u32(&s.o_full), 1);
    mbar_init(smem_u32(&s.o_free), 4);
    s.abort_flag = 0;
    fence_barrier_init();
  }
  // Dependent grids (the bf16 instance, the merge) may launch now; they wait
  // for this grid's completion.
  if (!kBf16) asm volatile("griddepcontrol.launch_dependents;");
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp < 4) {
    softmax_role<kD, kBf16>(s, p, tmem);
  } else if (warp == 4) {
    producer_role(s, p, &tmQ, &tmK, &tmV);
  } else if (warp == 5) {
    if (lane == 0) mma_role<kD, kBf16>(s, p, tmem);
  } else if (warp == 6) {
    prep_role<SharedStorage<kD>, kBf16>(s, p, p.bt);
  } else {
    convert_role<SharedStorage<kD>, kBf16>(s, p);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) {
    __syncwarp();
    tmem_dealloc(tmem, Geo<kD>::kTmemCols);
  }
  if (kBf16 && p.nsplit > 1) {
    // Every unit was claimed by ticket, so each is held by a running CTA: wait
    // (bounded) until all partials of the recomputed ranges are written, then
    // merge this CTA's share of the rows.
    if (threadIdx.x == 0) {
      const int want = SharedStorage<kD>::kSoftmaxWarps * p.BH * p.nparts;  // each softmax warp counts its rows
      const volatile int* cnt = &p.counters[kCtrParts];
      const uint64_t t0 = globaltimer_ns();
      while (*cnt < want) {
        if ((*reinterpret_cast<volatile uint32_t*>(p.status) & kStatusTimeout) ||
            globaltimer_ns() - t0 > kWaitTimeoutNs) {
          atomicOr(p.status, kStatusTimeout);
          break;
        }
        __nanosleep(256);
      }
      __threadfence();
    }
    __syncthreads();
    merge_ranges<kD, kThreads>(p, blockIdx.x, gridDim.x);
  }
  // The CTA that finishes last puts the workspace counters back to zero for
  // the next call (every other CTA is done with them).
  // (The flag is left for the bf16 instance, which clears it when it runs.)
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&p.counters[kCtrDone], 1) == static_cast<int>(gridDim.x) - 1) {
      p.counters[kCtrTickets] = 0;
      p.counters[kCtrDone] = 0;
      if (kBf16) {
        p.counters[kCtrBigV] = 0;
        p.counters[kCtrParts] = 0;
      }
    }
  }
}

// The split-row kernel at d = 64 (fp16 instance, or the bf16 instance with
// the merge of the global rows' ranges): the same units, scheduling, workspace
// and bf16 recompute as bigbird_fwd_kernel, with 12 warps -- 0..7 softmax
// (two per row), 8 TMA, 9 MMA (and TMEM), 10 unit preparation, 11 V
// conversion -- and two CTAs per SM.
template <bool kBf16>
__global__ void __launch_bounds__(kThreads2, 2)
bigbird_fwd2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ OutMaps tmO,
                    const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  SharedStorage2& s =
      *reinterpret_cast<SharedStorage2*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (kBf16) {
    // Merge the fp16 instance's ranges at once (the flag's load overlaps the
    // merge); when the flag is set the call is redone and merged again.
    asm volatile("griddepcontrol.launch_dependents;");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    int big_v = 0;
    if (threadIdx.x == 0) big_v = *reinterpret_cast<volatile int*>(&p.counters[kCtrBigV]);
    if (p.nsplit > 1) merge_ranges<64, kThreads2>(p, blockIdx.x, gridDim.x);
    if (threadIdx.x == 0) s.abort_flag = big_v;
    __syncthreads();
    if (s.abort_flag == 0) return;
    __syncthreads();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(&s.tmem_base), kTmemCols2);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(smem_u32(&s.info_full[i]), 1);
      mbar_init(smem_u32(&s.info_empty[i]), 1 + 1 + 8 + 1);  // TMA, MMA, 8 softmax warps, converter
    }
    for (int i = 0; i < SharedStorage2::kQBufs; ++i) {
      mbar_init(smem_u32(&s.q_full[i]), 1);
      mbar_init(smem_u32(&s.q_free[i]), 1);
    }
    for (int i = 0; i < SharedStorage2::kKSt; ++i) {
      mbar_init(smem_u32(&s.k_full[i]), 1);
      mbar_init(smem_u32(&s.k_empty[i]), 1);
    }
    for (int i = 0; i < SharedStorage2::kVSt; ++i) {
      mbar_init(smem_u32(&s.v_full[i]), 1);
      mbar_init(smem_u32(&s.v_conv[i]), 1);
      mbar_init(smem_u32(&s.v_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s.s_full[i]), 1);
      mbar_init(smem_u32(&s.p_full[i]), 8 + 1);  // eight softmax warps and the converter
      mbar_init(smem_u32(&s.pv_done[i]), 1);
    }
    mbar_init(smem_u32(&s.o_full), 1);
    mbar_init(smem_u32(&s.o_free), 8);
    mbar_init(smem_u32(&s.ml_ready), 8);
    mbar_init(smem_u32(&s.tile_ready), 8);
    s.abort_flag = 0;
    fence_barrier_init();
  }
  // The dependent grid (the bf16 instance) may launch now; it waits for this
  // grid's completion.
  if (!kBf16) asm volatile("griddepcontrol.launch_dependents;");
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO.out);
    if (p.nsplit > 1) tma_prefetch_desc(&tmO.part);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp < 8) {
    softmax2_role<kBf16>(s, p, tmem, &tmO);
    // the bf16 output tiles' TMA stores read shared memory until they complete
    if (warp == 0 && lane == 0) bulk_wait_all();
  } else if (warp == 8) {
    producer_role(s, p, &tmQ, &tmK, &tmV);
  } else if (warp == 9) {
    if (lane == 0) mma2_role<kBf16>(s, p, tmem);
  } else if (warp == 10) {
    prep_role<SharedStorage2, kBf16>(s, p, p.bt);
  } else {
    convert_role<SharedStorage2, kBf16>(s, p);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols2);
  }
  if (kBf16 && p.nsplit > 1) {
    // Every unit was claimed by ticket, so each is held by a running CTA: wait
    // (bounded) until all partials of the recomputed ranges are written, then
    // merge this CTA's share of the rows.
    if (threadIdx.x == 0) {
      const int want = SharedStorage2::kSoftmaxWarps * p.BH * p.nparts;  // each softmax warp counts its rows
      const volatile int* cnt = &p.counters[kCtrParts];
      const uint64_t t0 = globaltimer_ns();
      while (*cnt < want) {
        if ((*reinterpret_cast<volatile uint32_t*>(p.status) & kStatusTimeout) ||
            globaltimer_ns() - t0 > kWaitTimeoutNs) {
          atomicOr(p.status, kStatusTimeout);
          break;
        }
        __nanosleep(256);
      }
      __threadfence();
    }
    __syncthreads();
    merge_ranges<64, kThreads2>(p, blockIdx.x, gridDim.x);
  }
  // The CTA that finishes last puts the workspace counters back to zero for
  // the next call (every other CTA is done with them).
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&p.counters[kCtrDone], 1) == static_cast<int>(gridDim.x) - 1) {
      p.counters[kCtrTickets] = 0;
      p.counters[kCtrDone] = 0;
      if (kBf16) {
        p.counters[kCtrBigV] = 0;
        p.counters[kCtrParts] = 0;
      }
    }
  }
}

// Self-test of the bounded-wait path: one thread waits for an mbarrier that
// nothing arrives on; the wait runs out after limit_ns and sets the timeout
// bit of the status word, as a lost completion inside the forward would.
__global__ void bigbird_wait_probe_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
    if (!mbar_wait_for(smem_u32(&bar), 0, limit_ns)) atomicOr(status, kStatusTimeout);
  }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// Tensor map over [rows, 64] bf16 with 64x64 boxes and 128-byte swizzle.
// Tensor map over a [rows, d] bf16 matrix with 64x64 boxes (64 rows, one
// 64-column chunk) and 128-byte swizzle.
static bool make_map(CUtensorMap* map, const void* base, uint64_t rows, int d) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(kBlock)};
  const cuuint32_t es[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DeviceInfo {
  int sms = 0;
  bool ok = false;
  bool attr_set = false;
  uint32_t* status = nullptr;  // device address of g_status on this device
};

static DeviceInfo* device_info(int dev) {
  static DeviceInfo infos[64];
  static std::mutex mu;
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  DeviceInfo& di = infos[dev];
  if (!di.attr_set) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return nullptr;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return nullptr;
    di.ok = (major == 10);
    di.sms = sms;
    if (di.ok) {
      // Two CTAs per SM (either kernel) need the largest shared-memory carve-out.
      const struct {
        const void* fn;
        int smem;
      } kernels[] = {
          {reinterpret_cast<const void*>(bigbird_fwd_kernel<128, false>), static_cast<int>(sizeof(SharedStorage<128>) + 1024)},
          {reinterpret_cast<const void*>(bigbird_fwd_kernel<128, true>), static_cast<int>(sizeof(SharedStorage<128>) + 1024)},
          {reinterpret_cast<const void*>(bigbird_fwd2_kernel<false>), static_cast<int>(sizeof(SharedStorage2) + 1024)},
          {reinterpret_cast<const void*>(bigbird_fwd2_kernel<true>), static_cast<int>(sizeof(SharedStorage2) + 1024)},
      };
      for (const auto& kf : kernels) {
        if (cudaFuncSetAttribute(kf.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kf.smem) != cudaSuccess)
          return nullptr;
        if (cudaFuncSetAttribute(kf.fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
          return nullptr;
      }
      if (cudaGetSymbolAddress(reinterpret_cast<void**>(&di.status), g_status) != cudaSuccess) return nullptr;
    }
    di.attr_set = true;
  }
  return &di;
}

bool make_tile_map(CUtensorMap* map, const void* base, uint64_t rows) { return make_map(map, base, rows, 64); }
bool make_tile_map_d(CUtensorMap* map, const void* base, uint64_t rows, int d) { return make_map(map, base, rows, d); }

bool make_f32_map(CUtensorMap* map, const void* base, uint64_t rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {64 * 4};
  const cuuint32_t box[2] = {32u, static_cast<cuuint32_t>(kBlock)};
  const cuuint32_t es[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

uint32_t* status_word(int dev) {
  DeviceInfo* di = device_info(dev);
  return di && di->ok ? di->status : nullptr;
}


struct Plan {
  int nb = 0;
  int nt = 0;
  int bt = 1;
  bool sparse = false;
  int nsplit = 1;
  int split_tiles = 0;
  int n_glob = 1;
  size_t ws_bytes = 0;
};

// Blocks of 64 or 128 tokens at d = 64 or 128 run on this kernel; other sizes return
// BB_ERR_UNSUPPORTED here (the caller then tries the CUDA-core kernel).
static int make_plan(int B, int H, int L, int d, int block, int r, unsigned flags, Plan& pl) {
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0 || block <= 0 || r < 1 || L % block != 0) return BB_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || (block != kBlock && block != 2 * kBlock) || r > kMaxR) return BB_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * L >= (int64_t(1) << 31)) return BB_ERR_UNSUPPORTED;
  pl.nb = L / block;
  pl.bt = block / kBlock;
  pl.nt = L / kBlock;
  pl.sparse = (flags & BB_FLAG_FORCE_SPARSE) || pl.nb > 5 + 2 * r;
  if (pl.sparse && pl.nb < 5 + r) return BB_ERR_INVALID_ARG;
  if (pl.sparse) {
    // a middle unit lists at most 6 + 2r tiles (block 64: two query blocks'
    // union) or 2 (5 + r) (block 128); both fit kMaxList for r <= kMaxR
    // longer ranges for long sequences: fewer partial results to write and
    // merge, while the many middle units still balance the grid's tail
    pl.split_tiles = (pl.bt == 1 && d == 64 && pl.nt >= 256) ? kSplitBlocksLong : kSplitBlocks;
    pl.nsplit = (pl.nt + pl.split_tiles - 1) / pl.split_tiles;
    pl.n_glob = pl.bt == 1 ? 1 : 2;
  } else {
    // full attention in one range: nt <= (5 + 2r) bt tiles must fit the list
    if (pl.nt > kMaxList) return BB_ERR_UNSUPPORTED;
    pl.split_tiles = pl.nt;
    pl.nsplit = 1;
    pl.n_glob = 1;
  }
  // Workspace: the counters (unit tickets, finished CTAs, the bf16 flag),
  // then (split global rows only) the partial outputs [B*H, n_glob*nsplit,
  // 128, d] and their (max, sum) [B*H, n_glob*nsplit, 128, 2].
  pl.ws_bytes = kCounterBytes;
  if (pl.nsplit > 1)
    pl.ws_bytes += static_cast<size_t>(B) * H * pl.n_glob * pl.nsplit * kRows * (d + 2) * sizeof(float);
  return BB_OK;
}

// The launches of one call at head dimension kD: the fp16 instance, then the
// bf16 instance (which also merges split global rows) as its programmatic
// dependent: launched while the fp16 grid runs, it waits
// (griddepcontrol.wait) for that grid's completion before it reads what the
// grid wrote, which hides the launch gap.
template <int kD>
static cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                              int sms, cudaStream_t stream) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  const int grid = std::min(p.total_units, Geo<kD>::kCtasPerSm * sms);
  const size_t smem = sizeof(SharedStorage<kD>) + 1024;
  bigbird_fwd_kernel<kD, false><<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, bigbird_fwd_kernel<kD, true>, tq, tk, tv, p);
  }
  return e;
}

// The d = 64 launches: the split-row kernel's fp16 instance, then its bf16
// instance as the programmatic dependent (as in launch_fwd).
static cudaError_t launch_fwd2(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const OutMaps& to, const FwdParams& p, int sms, cudaStream_t stream) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  const int grid = std::min(p.total_units, 2 * sms);
  const size_t smem = sizeof(SharedStorage2) + 1024;
  bigbird_fwd2_kernel<false><<<grid, kThreads2, smem, stream>>>(tq, tk, tv, to, p);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads2);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, bigbird_fwd2_kernel<true>, tq, tk, tv, to, p);
  }
  return e;
}

}  // namespace bb

using namespace bb;

extern "C" {

size_t bigbird_attn_workspace_size(int B, int H, int L, int d, int block, int r, unsigned flags) {
  Plan pl;
  if (make_plan(B, H, L, d, block, r, flags, pl) != BB_OK) return 0;
  return pl.ws_bytes;
}

static int fwd_impl(const void* q, const void* k, const void* v, const int32_t* rand_attn, const uint8_t* seq_mask,
                    void* out, float* lse, int B, int H, int L, int d, int block, int r, int out_dtype, unsigned flags,
                    void* workspace, size_t workspace_bytes, void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  Plan pl;
  int st = make_plan(B, H, L, d, block, r, flags, pl);
  // Other supported sizes run the CUDA-core kernel (no workspace).
  if (st == BB_ERR_UNSUPPORTED && generic_fwd_supported(d, block))
    return generic_fwd(q, k, v, rand_attn, seq_mask, out, lse, B, H, L, d, block, r, out_dtype, flags, stream_);
  if (st != BB_OK) return st;
  if (!q || !k || !v || !out) return BB_ERR_INVALID_ARG;
  if (pl.sparse && !rand_attn) return BB_ERR_INVALID_ARG;
  if (out_dtype != BB_OUT_BF16 && out_dtype != BB_OUT_F32) return BB_ERR_INVALID_ARG;
  auto misaligned = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) != 0; };
  if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(out, 16)) return BB_ERR_UNSUPPORTED;
  if (workspace && (misaligned(workspace, 256) || workspace_bytes < pl.ws_bytes)) return BB_ERR_INVALID_ARG;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BB_ERR_CUDA;
  DeviceInfo* di = device_info(dev);
  if (!di) return BB_ERR_CUDA;
  if (!di->ok) return BB_ERR_UNSUPPORTED;

  if (pl.sparse && (flags & BB_FLAG_DEBUG_CHECKS)) {
    const size_t n = static_cast<size_t>(H) * (pl.nb - 2) * r;
    int32_t* h = static_cast<int32_t*>(malloc(n * sizeof(int32_t)));
    if (!h) return BB_ERR_CUDA;
    cudaError_t e = cudaMemcpyAsync(h, rand_attn, n * sizeof(int32_t), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    int vs = e == cudaSuccess ? bigbird_rand_attn_validate(h, H, L, block, r, 0) : BB_ERR_CUDA;
    free(h);
    if (vs != BB_OK) return vs;
  }

  CUtensorMap tq, tk, tv;
  const uint64_t rows = static_cast<uint64_t>(B) * H * L;
  if (!make_map(&tq, q, rows, d) || !make_map(&tk, k, rows, d) || !make_map(&tv, v, rows, d)) return BB_ERR_CUDA;

  FwdParams p{};
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.rand_attn = rand_attn;
  p.seq_mask = seq_mask;
  p.out = out;
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.L = L;
  p.nb = pl.nb;
  p.r = r;
  p.BH = B * H;
  p.sparse = pl.sparse ? 1 : 0;
  p.nt = pl.nt;
  p.bt = pl.bt;
  p.nsplit = pl.nsplit;
  p.split_tiles = pl.split_tiles;
  p.n_glob = pl.n_glob;
  p.nparts = pl.n_glob * pl.nsplit;
  if (pl.sparse) {
    // middle units: pairs of query blocks (block 64) or single blocks (block 128)
    p.n_pairs = pl.bt == 1 ? (pl.nb - 2 + 1) / 2 : pl.nb - 2;
    p.n_pair_units = p.BH * p.n_pairs;
    p.total_units = p.n_pair_units + p.BH * p.nparts;
  } else {
    p.n_pairs = 0;
    p.n_pair_units = 0;
    p.total_units = p.BH * ((pl.nt + 1) / 2);
  }
  p.out_f32 = out_dtype == BB_OUT_F32 ? 1 : 0;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(d));
  p.bias_raw = -10000.0f * sqrtf(static_cast<float>(d));

  p.status = di->status;

  void* ws = workspace;
  bool owned = false;
  if (!ws) {
    if (cudaMallocAsync(&ws, pl.ws_bytes, stream) != cudaSuccess) return BB_ERR_CUDA;
    owned = true;
    // a fresh workspace's counters start at zero
    if (cudaMemsetAsync(ws, 0, kCounterBytes, stream) != cudaSuccess) {
      cudaFreeAsync(ws, stream);
      return BB_ERR_CUDA;
    }
  }
  p.counters = static_cast<int*>(ws);
  if (pl.nsplit > 1) {
    p.part_o = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kCounterBytes);
    p.part_ml = p.part_o + static_cast<size_t>(p.BH) * p.nparts * kRows * d;
  }
  cudaError_t e = cudaSuccess;
  if (d == 64) {
    // the split-row kernel's output tiles leave through TMA stores: out (bf16
    // 64x64 boxes, or fp32 64-row x 32-column boxes) and the ranges' partials
    OutMaps om;
    bool ok = p.out_f32 ? make_f32_map(&om.out, out, rows) : make_map(&om.out, out, rows, 64);
    if (ok && pl.nsplit > 1) ok = make_f32_map(&om.part, p.part_o, static_cast<uint64_t>(p.BH) * p.nparts * kRows);
    else om.part = om.out;  // not used
    e = ok ? launch_fwd2(tq, tk, tv, om, p, di->sms, stream) : cudaErrorInvalidValue;
  } else {
    e = launch_fwd<128>(tq, tk, tv, p, di->sms, stream);
  }
  if (owned) cudaFreeAsync(ws, stream);
  return e == cudaSuccess ? BB_OK : BB_ERR_CUDA;
}

int bigbird_attn_fwd_ex(const void* q, const void* k, const void* v, const int32_t* rand_attn,
                        const uint8_t* seq_mask, void* out, int B, int H, int L, int d, int block, int r,
                        int out_dtype, unsigned flags, void* workspace, size_t workspace_bytes, void* stream) {
  return fwd_impl(q, k, v, rand_attn, seq_mask, out, nullptr, B, H, L, d, block, r, out_dtype, flags, workspace,
                  workspace_bytes, stream);
}

int bigbird_attn_fwd_train(const void* q, const void* k, const void* v, const int32_t* rand_attn,
                           const uint8_t* seq_mask, void* out, float* lse, int B, int H, int L, int d, int block,
                           int r, int out_dtype, unsigned flags, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (!lse) return BB_ERR_INVALID_ARG;
  return fwd_impl(q, k, v, rand_attn, seq_mask, out, lse, B, H, L, d, block, r, out_dtype, flags, workspace,
                  workspace_bytes, stream);
}

int bigbird_attn_fwd(const void* q, const void* k, const void* v, const int32_t* rand_attn, const uint8_t* seq_mask,
                     void* out, int B, int H, int L, int d, int block, int r, void* stream) {
  return bigbird_attn_fwd_ex(q, k, v, rand_attn, seq_mask, out, B, H, L, d, block, r, BB_OUT_BF16, 0u, nullptr, 0,
                             stream);
}

int bigbird_wait_probe(unsigned limit_us, void* stream_) {
  if (limit_us == 0 || limit_us > 2000000u) return BB_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BB_ERR_CUDA;
  DeviceInfo* di = device_info(dev);
  if (!di || !di->status) return BB_ERR_CUDA;
  bigbird_wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream_)>>>(
      di->status, static_cast<uint64_t>(limit_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? BB_OK : BB_ERR_CUDA;
}

int bigbird_device_status(void* stream_, uint32_t* host_status) {
  if (!host_status) return BB_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return BB_ERR_CUDA;
  uint32_t zero = 0;
  if (cudaMemcpyFromSymbol(host_status, g_status, sizeof(uint32_t)) != cudaSuccess) return BB_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(uint32_t)) != cudaSuccess) return BB_ERR_CUDA;
  return BB_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- no-allocation entry point
//
// Some callers cannot allocate device memory while they run this op: an
// inference server or real-time pipeline that reserves all device memory at
// start-up and forbids allocation (and the device-wide synchronisation that
// cudaMalloc/cudaFree can cause) inside its steady-state loop. For them,
// bigbird_attn_fwd_noalloc uses this fixed scratch region, which lives in the
// library's module: every GPU that loads the library holds it until the
// process exits.

namespace bb {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on device `dev` (which must be current).
// The host-side name is only a stand-in for the symbol: a kernel must be given
// this looked-up address, never &g_static_scratch. Looked up once per device.
static void* static_scratch_address(int dev) {
  static void* addr[64];
  static std::once_flag once[64];
  if (dev < 0 || dev >= 64) return nullptr;
  std::call_once(once[dev], [dev] {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) == cudaSuccess) addr[dev] = ptr;
  });
  return addr[dev];
}

}  // namespace bb

extern "C" int bigbird_attn_fwd_noalloc(const void* q, const void* k, const void* v, const int32_t* rand_attn,
                                        const uint8_t* seq_mask, void* out, int B, int H, int L, int d, int block,
                                        int r, int out_dtype, unsigned flags, void* stream) {
  // The debug checks copy rand_attn into a host buffer that they allocate.
  if (flags & BB_FLAG_DEBUG_CHECKS) return BB_ERR_UNSUPPORTED;
  bb::Plan pl;
  const int st = bb::make_plan(B, H, L, d, block, r, flags, pl);
  // The CUDA-core kernel for other sizes needs no scratch.
  if (st == BB_ERR_UNSUPPORTED && bb::generic_fwd_supported(d, block))
    return bigbird_attn_fwd_ex(q, k, v, rand_attn, seq_mask, out, B, H, L, d, block, r, out_dtype, flags, nullptr, 0,
                               stream);
  if (st != BB_OK) return st;
  if (pl.ws_bytes > bb::kStaticScratchBytes) return BB_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BB_ERR_CUDA;
  void* scratch = bb::static_scratch_address(dev);
  if (!scratch) return BB_ERR_CUDA;
  // The region keeps whatever the previous call left; the counters must start
  // at zero (a call that completes leaves them so, one that gave up may not).
  if (cudaMemsetAsync(scratch, 0, bb::kCounterBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return BB_ERR_CUDA;
  return bigbird_attn_fwd_ex(q, k, v, rand_attn, seq_mask, out, B, H, L, d, block, r, out_dtype, flags, scratch,
                             bb::kStaticScratchBytes, stream);
}

extern "C" size_t bigbird_attn_noalloc_scratch_bytes(void) { return bb::kStaticScratchBytes; }

// ------------------------------------------------------------ host buffers

// bigbird_attn_fwd_host: inputs and output in host memory. The batch is
// processed one sequence at a time through two device slots, on three
// streams of the library's own (host-to-device copies, the forward, device-to-
// host copies), so that copying sequence b+1 in, computing b and copying b-1
// out overlap; the caller's stream waits for the whole call at the end.

namespace bb {

struct HostPipe {
  std::mutex mu;  // one call at a time enqueues on the device's streams and events
  cudaStream_t h2d = nullptr, comp = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, in_done[2] = {}, comp_done[2] = {}, out_done[2] = {}, finish = nullptr;
  bool ok = false;
};

static HostPipe* host_pipe(int dev) {
  static HostPipe pipes[64];
  static std::once_flag once[64];
  if (dev < 0 || dev >= 64) return nullptr;
  std::call_once(once[dev], [dev] {
    HostPipe& hp = pipes[dev];
    bool ok = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.comp, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.finish, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; i < 2 && ok; ++i)
      ok = cudaEventCreateWithFlags(&hp.in_done[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.comp_done[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.out_done[i], cudaEventDisableTiming) == cudaSuccess;
    hp.ok = ok;
  });
  return pipes[dev].ok ? &pipes[dev] : nullptr;
}

struct HostLayout {
  size_t ra = 0, slot = 0, q = 0, k = 0, v = 0, out = 0, mask = 0, ws = 0, ws_bytes = 0, total = 0;
};

static size_t r256(size_t x) { return (x + 255) / 256 * 256; }

// Scratch layout: rand_attn, then two slots of one sequence's q, k, v, out
// (fp32-sized), seq_mask and forward workspace. 0 if the sizes are invalid.
static bool host_layout(int B, int H, int L, int d, int block, int r, unsigned flags, HostLayout& hl) {
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0 || block <= 0 || r < 1 || L % block != 0) return false;
  const size_t rows = static_cast<size_t>(H) * L;
  const int nb = L / block;
  hl.ws_bytes = bigbird_attn_workspace_size(1, H, L, d, block, r, flags);
  hl.ra = 0;
  size_t off = r256(static_cast<size_t>(H) * (nb > 2 ? nb - 2 : 1) * r * sizeof(int32_t));
  hl.q = 0;
  hl.k = r256(rows * d * 2);
  hl.v = hl.k + r256(rows * d * 2);
  hl.out = hl.v + r256(rows * d * 2);
  hl.mask = hl.out + r256(rows * d * 4);
  hl.ws = hl.mask + r256(static_cast<size_t>(L));
  hl.slot = hl.ws + r256(hl.ws_bytes);
  hl.total = off + 2 * hl.slot;
  hl.ra = 0;
  // slot s starts at off + s * slot
  hl.q += off;
  hl.k += off;
  hl.v += off;
  hl.out += off;
  hl.mask += off;
  hl.ws += off;
  return true;
}

}  // namespace bb

extern "C" size_t bigbird_attn_fwd_host_scratch_bytes(int B, int H, int L, int d, int block, int r, unsigned flags) {
  bb::HostLayout hl;
  return bb::host_layout(B, H, L, d, block, r, flags, hl) ? hl.total : 0;
}

extern "C" int bigbird_attn_fwd_host(const void* q, const void* k, const void* v, const int32_t* rand_attn,
                                     const uint8_t* seq_mask, void* out, int B, int H, int L, int d, int block, int r,
                                     int out_dtype, unsigned flags, void* scratch, size_t scratch_bytes,
                                     void* stream_) {
  using namespace bb;
  HostLayout hl;
  if (!host_layout(B, H, L, d, block, r, flags, hl)) return BB_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !scratch) return BB_ERR_INVALID_ARG;
  if (out_dtype != BB_OUT_BF16 && out_dtype != BB_OUT_F32) return BB_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(scratch) & 255) != 0 || scratch_bytes < hl.total) return BB_ERR_INVALID_ARG;
  const int nb = L / block;
  const bool sparse = (flags & BB_FLAG_FORCE_SPARSE) || nb > 5 + 2 * r;
  if (sparse && !rand_attn) return BB_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BB_ERR_CUDA;
  HostPipe* hp = host_pipe(dev);
  if (!hp) return BB_ERR_CUDA;
  std::lock_guard<std::mutex> lock(hp->mu);
  cudaStream_t caller = static_cast<cudaStream_t>(stream_);
  uint8_t* base = static_cast<uint8_t*>(scratch);
  const size_t seq_in = static_cast<size_t>(H) * L * d * 2;
  const size_t seq_out = static_cast<size_t>(H) * L * d * (out_dtype == BB_OUT_F32 ? 4 : 2);
  // everything already queued on the caller's stream (earlier users of the
  // scratch) comes first
  if (cudaEventRecord(hp->start, caller) != cudaSuccess) return BB_ERR_CUDA;
  for (cudaStream_t s : {hp->h2d, hp->comp, hp->d2h})
    if (cudaStreamWaitEvent(s, hp->start, 0) != cudaSuccess) return BB_ERR_CUDA;
  int32_t* ra_d = reinterpret_cast<int32_t*>(base + hl.ra);
  if (sparse && cudaMemcpyAsync(ra_d, rand_attn, static_cast<size_t>(H) * (nb - 2) * r * sizeof(int32_t),
                                cudaMemcpyHostToDevice, hp->h2d) != cudaSuccess)
    return BB_ERR_CUDA;
  // a fresh call's workspace counters start at zero
  for (int sl = 0; sl < 2; ++sl)
    if (hl.ws_bytes && cudaMemsetAsync(base + sl * hl.slot + hl.ws, 0, kCounterBytes, hp->h2d) != cudaSuccess)
      return BB_ERR_CUDA;
  int st = BB_OK;
  for (int b = 0; b < B && st == BB_OK; ++b) {
    const int sl = b & 1;
    uint8_t* slot = base + sl * hl.slot;
    // slot sl is free once sequence b-2 has been copied out
    if (b >= 2 && cudaStreamWaitEvent(hp->h2d, hp->out_done[sl], 0) != cudaSuccess) return BB_ERR_CUDA;
    const size_t off = static_cast<size_t>(b) * seq_in;
    if (cudaMemcpyAsync(slot + hl.q, static_cast<const uint8_t*>(q) + off, seq_in, cudaMemcpyHostToDevice, hp->h2d) !=
            cudaSuccess ||
        cudaMemcpyAsync(slot + hl.k, static_cast<const uint8_t*>(k) + off, seq_in, cudaMemcpyHostToDevice, hp->h2d) !=
            cudaSuccess ||
        cudaMemcpyAsync(slot + hl.v, static_cast<const uint8_t*>(v) + off, seq_in, cudaMemcpyHostToDevice, hp->h2d) !=
            cudaSuccess)
      return BB_ERR_CUDA;
    if (seq_mask && cudaMemcpyAsync(slot + hl.mask, seq_mask + static_cast<size_t>(b) * L, static_cast<size_t>(L),
                                    cudaMemcpyHostToDevice, hp->h2d) != cudaSuccess)
      return BB_ERR_CUDA;
    if (cudaEventRecord(hp->in_done[sl], hp->h2d) != cudaSuccess) return BB_ERR_CUDA;
    if (cudaStreamWaitEvent(hp->comp, hp->in_done[sl], 0) != cudaSuccess) return BB_ERR_CUDA;
    st = bigbird_attn_fwd_ex(slot + hl.q, slot + hl.k, slot + hl.v, sparse ? ra_d : nullptr,
                             seq_mask ? slot + hl.mask : nullptr, slot + hl.out, 1, H, L, d, block, r, out_dtype,
                             flags & ~static_cast<unsigned>(BB_FLAG_DEBUG_CHECKS),
                             hl.ws_bytes ? slot + hl.ws : nullptr, hl.ws_bytes, hp->comp);
    if (st != BB_OK) break;
    if (cudaEventRecord(hp->comp_done[sl], hp->comp) != cudaSuccess) return BB_ERR_CUDA;
    if (cudaStreamWaitEvent(hp->d2h, hp->comp_done[sl], 0) != cudaSuccess) return BB_ERR_CUDA;
    if (cudaMemcpyAsync(static_cast<uint8_t*>(out) + static_cast<size_t>(b) * seq_out, slot + hl.out, seq_out,
                        cudaMemcpyDeviceToHost, hp->d2h) != cudaSuccess)
      return BB_ERR_CUDA;
    if (cudaEventRecord(hp->out_done[sl], hp->d2h) != cudaSuccess) return BB_ERR_CUDA;
  }
  // the caller's stream waits for the last copy out (and so for everything)
  if (cudaEventRecord(hp->finish, hp->d2h) != cudaSuccess) return BB_ERR_CUDA;
  if (cudaStreamWaitEvent(caller, hp->finish, 0) != cudaSuccess) return BB_ERR_CUDA;
  return st;
}
