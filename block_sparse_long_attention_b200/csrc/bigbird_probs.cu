// Attention probabilities of BigBird ITC block-sparse attention for B200
// (sm_100a): the output_attentions path.
//
// The block-sparse model computes the weights of each row group and writes
// them into a full (batch, heads, L, L) matrix, zero outside the pattern
// [HF-Pegasus, section "三类注意力组合": four scatter_ calls]; that matrix is
// mostly zeros and carries no gradient [HF-Pegasus, section "使用限制与注意事项"].
// This kernel recomputes each listed 64x64 tile of scores and turns it into
// weights with the row log-sum-exp that the forward wrote
// (bigbird_attn_fwd_train): p = exp(s - lse). Every tile is produced on its
// own, in one pass, with no reduction across tiles.
//
// Layouts (fp32 or bf16):
//   packed  global rows [B, H, G, 64, L] (G = 2: query blocks 0 and nb-1; in
//           the full-attention fallback G = nb, i.e. the whole matrix) and
//           band tiles [B, H, nb-2, 5+r, 64, 64]: tile t of query block i is
//           its weights against key block list[t], where list is the row's
//           sorted distinct key blocks (bigbird_pattern_table's order); the
//           tiles past the end of the list are zero;
//   dense   [B, H, L, L], zero outside the pattern.
//
// A unit is one query block against up to 8 key-block tiles: a range of 8
// blocks of a full row, a row's band list (packed), or a range of 8 blocks of
// any row with its unlisted tiles zero (dense). The kernel is persistent
// (four CTAs of 320 threads per SM, units dealt out evenly) and
// warp-specialised, so one unit's setup, loads and MMAs overlap the previous
// unit's stores:
//   warp 8     plans each unit with all 32 lanes (its tiles and output
//              offsets; the band list from rand_attn, sorted and deduplicated
//              with shuffles) into a 2-slot ring, and loads the Q block and
//              the listed K tiles by TMA into 2-deep rings;
//   warp 9     TMEM allocation and the MMAs: scores transposed, S^T = K Q^T,
//              two key tiles at a time (M = 128 keys, N = 64 queries, four
//              tcgen05 128x64x16 steps) into one of two 64-column TMEM
//              buffers;
//   warps 0-7  thread (warp w, lane l) reads TMEM lane 32 (w % 4) + l (one
//              key) and the 32 query columns of half w / 4, 16 at a time,
//              and writes p for them. Consecutive lanes hold consecutive keys, so each store
//              instruction of a warp covers 32 consecutive elements of one
//              output row (128 bytes in fp32) with no shuffle. Zero tiles are
//              written with 16-byte stores.
// Output stores are streaming (evict-first); Q and K loads are kept in L2
// (each K block is read by every unit that lists it).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/bigbird_attn.h"
#include "bb_internal.h"
#include "sm100_ptx.cuh"

namespace bbp {

using namespace bb;

constexpr int kBlock = 64;
constexpr int kDim = 64;
constexpr int kTiles = 8;                   // key-block tiles per unit
constexpr int kEpiWarps = 8;                // warps that turn scores into weights
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kProdWarp = kEpiWarps;        // planning + TMA
constexpr int kMmaWarp = kEpiWarps + 1;     // TMEM + MMA
constexpr int kThreads = kEpiThreads + 64;
constexpr int kCtasPerSm = 4;
constexpr int kKSlots = 2;                  // K ring depth (MMA groups of two key tiles)
constexpr int kLdCols = 16;                 // TMEM columns a weight thread reads at a time (keeps 4 CTAs within 48 registers)
constexpr int kMaxR = 16;
constexpr uint32_t kTileBytes = kBlock * kDim * 2;
constexpr uint32_t kTmemCols = 128;         // two 64-column S^T buffers
constexpr uint32_t kStatusBadRandAttn = 1u;
constexpr uint32_t kStatusTimeout = 2u;
constexpr float kLog2e = 1.4426950408889634f;

struct ProbsParams {
  const float* lse;          // [B*H*L] natural-log log-sum-exp of each row's scores
  const int32_t* rand_attn;  // [H, nb-2, r]
  const uint8_t* seq_mask;   // [B, L], 1 = valid key, or null
  void* out_rows;            // packed: [B, H, G, 64, L]; dense: [B, H, L, L]
  void* out_band;            // packed: [B, H, nb-2, 5+r, 64, 64]
  uint32_t* status;
  int H, L, nb, r;
  int sparse;          // sparse pattern (else full attention)
  int dense;           // dense [B, H, L, L] layout
  int out_f32;
  int ranges;          // ranges of kTiles key blocks per row
  int chunks;          // band chunks of kTiles slots per row (packed)
  int grows;           // full rows per head in the packed layout
  int units_per_head;
  int total_units;
  int units_per_cta;   // CTA c takes units [c * units_per_cta, (c + 1) * units_per_cta)
  float scale_log2;    // log2(e) / sqrt(d)
  float bias_log2;     // -10000 * log2(e): the masked-key bias in log2 units
};

struct UnitInfo {
  long long tile_off[kTiles];  // element offset of each tile's (0, 0) in its output
  int32_t tile_kb[kTiles];     // key block of each tile, or -1 for a zero tile
  int32_t comp_tile[kTiles];   // compute slot -> tile index
  int32_t n_tiles;             // < 0: no more units (every role leaves its loop)
  int32_t n_comp, ld, bh, qblk, band;
};

struct __align__(1024) Smem {
  uint8_t q[2][kTileBytes];     // Q block ring (SW128)
  uint8_t k[kKSlots][2][kTileBytes];  // K ring: each slot holds the two key tiles of one MMA group (M = 128)
  float nlse2[kBlock];          // -lse * log2(e) of the current unit's 64 rows (weight warps)
  UnitInfo info[2];
  uint64_t info_full[2], info_empty[2];
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[kKSlots], k_empty[kKSlots];
  uint64_t mma_done[2], tmem_free[2];
  uint32_t tmem_base;
  int32_t abort_flag;
};

__device__ __forceinline__ bool aborted(const Smem& sm) {
  return *reinterpret_cast<const volatile int32_t*>(&sm.abort_flag) != 0;
}

__device__ __forceinline__ void set_abort(Smem& sm, const ProbsParams& p) {
  atomicOr(p.status, kStatusTimeout);
  *reinterpret_cast<volatile int32_t*>(&sm.abort_flag) = 1;
}

// Plan of unit `unit`, computed by all 32 lanes of the calling warp with
// registers and shuffles only: its query block, tiles and output offsets.
// The key blocks of a band row i (1 <= i <= nb-2) of head h are the set
// {0, nb-1, i-1, i, i+1} and the row's random blocks, in ascending order:
// lane c holds candidate c (lanes 5 .. 4+r load rand_attn[h][i-1][c-5]), a
// candidate equal to one on a lower lane is a duplicate, and a distinct
// candidate's slot is the number of distinct candidates below it.
// Out-of-range random entries are skipped and reported in the status word.
__device__ void plan_unit_warp(const ProbsParams& p, UnitInfo& in, int unit, int lane) {
  constexpr unsigned kFull = 0xffffffffu;
  constexpr int kNone = 0x7fffffff;
  const int bh = unit / p.units_per_head;
  int w = unit - bh * p.units_per_head;
  const int h = bh % p.H;
  const long long L = p.L;
  int i, g = 0, kb0 = 0, s0 = 0, n_tiles, ld = p.L, band = 0;
  bool full;
  if (p.dense) {
    i = w / p.ranges;
    kb0 = (w - i * p.ranges) * kTiles;
    full = !p.sparse || i == 0 || i == p.nb - 1;
    n_tiles = min(kTiles, p.nb - kb0);
  } else if (w < p.grows * p.ranges) {
    g = w / p.ranges;
    kb0 = (w - g * p.ranges) * kTiles;
    i = p.sparse ? (g == 0 ? 0 : p.nb - 1) : g;
    full = true;
    n_tiles = min(kTiles, p.nb - kb0);
  } else {
    w -= p.grows * p.ranges;
    i = 1 + w / p.chunks;
    s0 = (w - (i - 1) * p.chunks) * kTiles;
    full = false;
    n_tiles = min(kTiles, 5 + p.r - s0);
    ld = kBlock;
    band = 1;
  }
  // band rows: the distinct candidates and their slots
  int cand = kNone;
  bool valid = false;
  int rank = 0;
  if (!full) {
    if (lane < 5) {
      cand = lane == 0 ? 0 : lane == 1 ? p.nb - 1 : i - 3 + lane;  // lanes 2, 3, 4: i-1, i, i+1
    } else if (lane < 5 + p.r) {
      const int x = p.rand_attn[(static_cast<long long>(h) * (p.nb - 2) + (i - 1)) * p.r + (lane - 5)];
      if (x >= 0 && x < p.nb) cand = x;
      else atomicOr(p.status, kStatusBadRandAttn);
    }
    bool dup = false;
    for (int o = 0; o < 5 + kMaxR; ++o) {
      const int v = __shfl_sync(kFull, cand, o);
      dup |= (o < lane && v == cand);
    }
    valid = cand != kNone && !dup;
    for (int o = 0; o < 5 + kMaxR; ++o) {
      const int v = __shfl_sync(kFull, cand, o);
      const bool vo = __shfl_sync(kFull, valid ? 1 : 0, o) != 0;
      rank += (vo && v < cand) ? 1 : 0;
    }
  }
  // tile t is lane t's: key block (or -1: a zero tile) and output offset
  int kb = -1;
  long long off = 0;
  if (lane < n_tiles) {
    if (p.dense) {
      kb = kb0 + lane;
      off = (static_cast<long long>(bh) * L + static_cast<long long>(i) * kBlock) * L + static_cast<long long>(kb) * kBlock;
    } else if (!band) {
      kb = kb0 + lane;
      off = (static_cast<long long>(bh) * p.grows + g) * kBlock * L + static_cast<long long>(kb) * kBlock;
    } else {
      off = ((static_cast<long long>(bh) * (p.nb - 2) + (i - 1)) * (5 + p.r) + s0 + lane) *
            static_cast<long long>(kBlock * kBlock);
    }
  }
  if (!full) {
    if (band) {
      // slot s0 + t holds the candidate of rank s0 + t
      for (int t = 0; t < kTiles; ++t) {
        const unsigned owner = __ballot_sync(kFull, valid && rank == s0 + t);
        const int v = __shfl_sync(kFull, cand, owner ? __ffs(owner) - 1 : 0);
        if (lane == t) kb = owner ? v : -1;
      }
    } else {
      // dense layout: block kb0 + t is computed only if it is in the row's set
      const unsigned hit = __reduce_or_sync(
          kFull, (valid && cand >= kb0 && cand < kb0 + n_tiles) ? (1u << (cand - kb0)) : 0u);
      if (lane < n_tiles && !((hit >> lane) & 1u)) kb = -1;
    }
  }
  const bool comp = lane < n_tiles && kb >= 0;
  const unsigned cmask = __ballot_sync(kFull, comp);
  if (lane < n_tiles) {
    in.tile_kb[lane] = kb;
    in.tile_off[lane] = off;
  }
  if (comp) in.comp_tile[__popc(cmask & ((1u << lane) - 1u))] = lane;
  if (lane == 0) {
    in.n_tiles = n_tiles;
    in.n_comp = __popc(cmask);
    in.ld = ld;
    in.bh = bh;
    in.qblk = i;
    in.band = band;
  }
  __syncwarp();
}

__device__ __forceinline__ void epi_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kEpiThreads) : "memory");
}

// Named barrier of the weight threads that also ORs a predicate over them:
// every thread gets the same answer.
__device__ __forceinline__ bool epi_bar_or(bool x) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(x)), "r"(kEpiThreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void tmem_ld_cols(uint32_t a, uint32_t (&r)[32]) { tmem_ld32(a, r); }
__device__ __forceinline__ void tmem_ld_cols(uint32_t a, uint32_t (&r)[16]) { tmem_ld16(a, r); }

// p for one key and N query rows: x = s log2(e)/sqrt(d) + (bias2 - lse2[q]),
// two rows per packed f32x2 operation; row q of the tile is LD elements
// after row q-1 (LD = 0: the runtime stride ld).
template <int N, int LD, bool F32>
__device__ __forceinline__ void emit(const uint32_t (&v)[N], const float* nlse2, float bias2, float scale, void* dst,
                                     long long ld) {
  const uint64_t scale2 = f2_pack(scale, scale);
  const uint64_t bias22 = f2_pack(bias2, bias2);
  const long long stride = LD ? LD : ld;
#pragma unroll
  for (int c = 0; c < N; c += 4) {
    const float4 nl = *reinterpret_cast<const float4*>(nlse2 + c);
    const uint64_t x01 = f2_fma(f2_pack(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), scale2,
                                f2_add(f2_pack(nl.x, nl.y), bias22));
    const uint64_t x23 = f2_fma(f2_pack(__uint_as_float(v[c + 2]), __uint_as_float(v[c + 3])), scale2,
                                f2_add(f2_pack(nl.z, nl.w), bias22));
    float x[4];
    f2_unpack(x01, x[0], x[1]);
    f2_unpack(x23, x[2], x[3]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float pr = ex2_approx(x[e]);
      if (F32)
        __stcs(reinterpret_cast<float*>(dst) + (c + e) * stride, pr);
      else
        __stcs(reinterpret_cast<unsigned short*>(dst) + (c + e) * stride,
               __bfloat16_as_ushort(__float2bfloat16_rn(pr)));
    }
  }
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
bigbird_probs_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const ProbsParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (warp == kProdWarp && lane == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sm.info_full[b]), 1);
      mbar_init(smem_u32(&sm.info_empty[b]), 2);  // the MMA thread and the weight warps
      mbar_init(smem_u32(&sm.q_full[b]), 1);
      mbar_init(smem_u32(&sm.q_empty[b]), 1);
      mbar_init(smem_u32(&sm.mma_done[b]), 1);
      mbar_init(smem_u32(&sm.tmem_free[b]), kEpiThreads);
    }
    for (int b = 0; b < kKSlots; ++b) {
      mbar_init(smem_u32(&sm.k_full[b]), 1);
      mbar_init(smem_u32(&sm.k_empty[b]), 1);
    }
    fence_barrier_init();
    sm.abort_flag = 0;
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int u0 = blockIdx.x * p.units_per_cta;
  const int u1 = min(p.total_units, u0 + p.units_per_cta);

  if (warp == kProdWarp) {
    // ------------------------------------------------------------ plan + TMA
    // The whole warp plans each unit; lane 0 waits on the rings and issues
    // the loads, and tells the other lanes when to stop.
    const uint64_t keep = l2_policy_evict_last();
    int iq = 0, gk = 0;  // Q blocks and K groups loaded so far (lane 0)
    for (int iu = 0;; ++iu) {
      const int u = u0 + iu;
      const int s = iu & 1;
      UnitInfo& in = sm.info[s];
      int stop = 0;
      if (lane == 0) {
        if (iu >= 2 && !mbar_wait(smem_u32(&sm.info_empty[s]), ((iu - 2) >> 1) & 1)) {
          set_abort(sm, p);
          stop = 1;
        } else if (u >= u1 || aborted(sm)) {
          in.n_tiles = -1;
          mbar_arrive(smem_u32(&sm.info_full[s]));
          stop = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, stop, 0)) break;
      plan_unit_warp(p, in, u, lane);  // ends with __syncwarp: lane 0 sees every lane's entries
      if (lane == 0) {
        mbar_arrive(smem_u32(&sm.info_full[s]));  // release: the plan is visible to the waiting roles
        const int nc = in.n_comp;
        if (nc > 0) {  // (a unit of zero tiles only loads nothing)
          const int row0 = in.bh * p.L;
          const int qs = iq & 1;
          bool ok = !(iq >= 2 && !mbar_wait(smem_u32(&sm.q_empty[qs]), ((iq - 2) >> 1) & 1));
          if (ok) {
            mbar_arrive_expect_tx(smem_u32(&sm.q_full[qs]), kTileBytes);
            tma_load_2d(smem_u32(sm.q[qs]), &tmQ, smem_u32(&sm.q_full[qs]), 0, row0 + in.qblk * kBlock, keep);
            ++iq;
          }
          for (int g = 0; ok && g < (nc + 1) / 2; ++g, ++gk) {
            const int ks = gk % kKSlots;
            if (gk >= kKSlots && !mbar_wait(smem_u32(&sm.k_empty[ks]), (gk / kKSlots - 1) & 1)) {
              ok = false;
              break;
            }
            const int nt = min(2, nc - 2 * g);
            mbar_arrive_expect_tx(smem_u32(&sm.k_full[ks]), static_cast<uint32_t>(nt) * kTileBytes);
            for (int t = 0; t < nt; ++t)
              tma_load_2d(smem_u32(sm.k[ks][t]), &tmK, smem_u32(&sm.k_full[ks]), 0,
                          row0 + in.tile_kb[in.comp_tile[2 * g + t]] * kBlock, keep);
          }
          if (!ok) {
            set_abort(sm, p);
            stop = 1;
          }
        }
      }
      if (__shfl_sync(0xffffffffu, stop, 0)) break;
    }
    if (lane == 0) {
      // No copy may still be in flight when the CTA exits: wait (bounded) for
      // the last loads of both rings.
      for (int j = max(0, iq - 2); j < iq; ++j) mbar_wait(smem_u32(&sm.q_full[j & 1]), (j >> 1) & 1);
      for (int j = max(0, gk - kKSlots); j < gk; ++j) mbar_wait(smem_u32(&sm.k_full[j % kKSlots]), (j / kKSlots) & 1);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t idesc = idesc_f32acc(2 * kBlock, kBlock, true, false);  // bf16 K . Q^T, M = 128, N = 64
      int iq = 0, gk = 0, gt = 0;  // Q blocks, K groups, TMEM groups consumed
      bool issued = false;
      for (int iu = 0;; ++iu) {
        const int s = iu & 1;
        if (!mbar_wait(smem_u32(&sm.info_full[s]), (iu >> 1) & 1)) {
          set_abort(sm, p);
          break;
        }
        const UnitInfo& in = sm.info[s];
        if (in.n_tiles < 0) break;
        const int nc = in.n_comp;
        if (nc > 0) {
          const int qs = iq & 1;
          bool ok = mbar_wait(smem_u32(&sm.q_full[qs]), (iq >> 1) & 1);
          for (int g = 0; ok && g < (nc + 1) / 2; ++g, ++gk, ++gt) {
            const int ks = gk % kKSlots;
            const int buf = gt & 1;
            ok = mbar_wait(smem_u32(&sm.k_full[ks]), (gk / kKSlots) & 1) &&
                 (gt < 2 || mbar_wait(smem_u32(&sm.tmem_free[buf]), ((gt - 2) >> 1) & 1));
            if (!ok) break;
            tc_fence_after();
            const uint32_t ka = smem_u32(sm.k[ks][0]);
            const uint32_t qa = smem_u32(sm.q[qs]);
#pragma unroll
            for (int kk = 0; kk < kDim / 16; ++kk)
              mma_ss(tmem + static_cast<uint32_t>(buf) * kBlock, sdesc_sw128(ka + kk * 32, 16, 1024),
                     sdesc_sw128(qa + kk * 32, 16, 1024), idesc, kk > 0 ? 1u : 0u);
            mma_commit(smem_u32(&sm.mma_done[buf]));
            mma_commit(smem_u32(&sm.k_empty[ks]));
            issued = true;
          }
          if (!ok) {
            set_abort(sm, p);
            break;
          }
          mma_commit(smem_u32(&sm.q_empty[qs]));
          ++iq;
        }
        mbar_arrive(smem_u32(&sm.info_empty[s]));
      }
      // Every MMA has completed before TMEM is released (bounded).
      if (issued && gt > 0) mbar_wait(smem_u32(&sm.mma_done[(gt - 1) & 1]), ((gt - 1) >> 1) & 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ weights
    // Every decision to leave the unit loop is taken jointly by the 256
    // weight threads (bar.red.or), so they always meet at the same named
    // barriers; a failed wait only skips work after that point.
    const int et = tid;                 // 0 .. 255
    const int quad = warp & 3;          // TMEM lanes 32 quad .. 32 quad + 31
    const int half = warp >> 2;         // query columns 32 half .. 32 half + 31
    const int m = 32 * quad + lane;     // key row of a 128-key MMA group
    const int kk = m & (kBlock - 1);
    const int esize = p.out_f32 ? 4 : 2;
    int gt = 0;
    for (int iu = 0;; ++iu) {
      const int s = iu & 1;
      const bool ok = !aborted(sm) && mbar_wait(smem_u32(&sm.info_full[s]), (iu >> 1) & 1);
      if (!ok && !aborted(sm)) set_abort(sm, p);
      const UnitInfo& in = sm.info[s];
      const bool leave = epi_bar_or(!ok || in.n_tiles < 0);  // also: every thread is done with the previous unit
      if (iu >= 1 && et == 0) mbar_arrive(smem_u32(&sm.info_empty[s ^ 1]));
      if (leave) break;
      const int nc = in.n_comp;
      const int ngroups = (nc + 1) / 2;
      uint8_t* out = static_cast<uint8_t*>(in.band ? p.out_band : p.out_rows);
      const long long ld = in.ld;
      if (et < kBlock) sm.nlse2[et] = -p.lse[static_cast<long long>(in.bh) * p.L + in.qblk * kBlock + et] * kLog2e;
      // which of this thread's keys (one per group) are padded; loads issued before any wait
      uint32_t masked = 0;
      if (p.seq_mask) {
        const uint8_t* sm_row = p.seq_mask + static_cast<long long>(in.bh / p.H) * p.L + kk;
#pragma unroll
        for (int g = 0; g < kTiles / 2; ++g) {
          const int cs = 2 * g + (m >> 6);
          if (cs < nc && !sm_row[in.tile_kb[in.comp_tile[cs]] * kBlock]) masked |= 1u << g;
        }
      }
      // zero tiles
      const int vec_per_row = kBlock * esize / 16;
      for (int t = 0; t < in.n_tiles; ++t) {
        if (in.tile_kb[t] >= 0) continue;
        uint8_t* base = out + in.tile_off[t] * esize;
        for (int idx = et; idx < kBlock * vec_per_row; idx += kEpiThreads) {
          const int row = idx / vec_per_row;
          const int col = idx - row * vec_per_row;
          __stcs(reinterpret_cast<uint4*>(base + (static_cast<long long>(row) * ld) * esize) + col,
                 make_uint4(0u, 0u, 0u, 0u));
        }
      }
      epi_bar_sync();  // nlse2 visible
      for (int g = 0; g < ngroups; ++g, ++gt) {
        const int buf = gt & 1;
        const bool okw = !aborted(sm) && mbar_wait(smem_u32(&sm.mma_done[buf]), (gt >> 1) & 1);
        if (__all_sync(0xffffffffu, okw)) {
          tc_fence_after();
          const int cs = 2 * g + (m >> 6);
          const bool act = cs < nc;
          const long long off = act ? in.tile_off[in.comp_tile[cs]] : 0;
          const float bias2 = (masked >> g) & 1u ? p.bias_log2 : 0.0f;
#pragma unroll
          for (int c0 = 0; c0 < 32; c0 += kLdCols) {
            uint32_t v[kLdCols];
            tmem_ld_cols(tmem + (static_cast<uint32_t>(32 * quad) << 16) +
                             static_cast<uint32_t>(buf * kBlock + 32 * half + c0), v);
            tmem_wait_ld();
            if (c0 + kLdCols == 32) {  // the buffer is fully read: the next MMA may overwrite it
              tc_fence_before();
              mbar_arrive(smem_u32(&sm.tmem_free[buf]));
            }
            if (act) {
              uint8_t* dst = out + (off + kk + static_cast<long long>(32 * half + c0) * ld) * esize;
              const float* nl = sm.nlse2 + 32 * half + c0;
              if (in.band) {
                if (p.out_f32) emit<kLdCols, kBlock, true>(v, nl, bias2, p.scale_log2, dst, ld);
                else emit<kLdCols, kBlock, false>(v, nl, bias2, p.scale_log2, dst, ld);
              } else {
                if (p.out_f32) emit<kLdCols, 0, true>(v, nl, bias2, p.scale_log2, dst, ld);
                else emit<kLdCols, 0, false>(v, nl, bias2, p.scale_log2, dst, ld);
              }
            }
          }
        } else {
          if (!aborted(sm)) set_abort(sm, p);
          mbar_arrive(smem_u32(&sm.tmem_free[buf]));
        }
      }
    }
  }

  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

struct Layout {
  int nb = 0;
  bool sparse = false;
  int grows = 0;       // full rows per head (packed)
  int band_rows = 0;   // nb - 2, or 0 in the fallback
  int band_slots = 0;  // 5 + r, or 0 in the fallback
};

static int make_layout(int L, int d, int block, int r, unsigned flags, Layout& lo) {
  if (L <= 0 || d <= 0 || block <= 0 || r < 1 || L % block != 0) return BB_ERR_INVALID_ARG;
  if (d != kDim || block != kBlock || r > kMaxR) return BB_ERR_UNSUPPORTED;
  lo.nb = L / block;
  lo.sparse = (flags & BB_FLAG_FORCE_SPARSE) || lo.nb > 5 + 2 * r;
  if (lo.sparse && lo.nb < 5 + r) return BB_ERR_INVALID_ARG;
  lo.grows = lo.sparse ? 2 : lo.nb;
  lo.band_rows = lo.sparse ? lo.nb - 2 : 0;
  lo.band_slots = lo.sparse ? 5 + r : 0;
  return BB_OK;
}

static int probs_impl(const void* q, const void* k, const float* lse, const int32_t* rand_attn,
                      const uint8_t* seq_mask, void* out_rows, void* out_band, int B, int H, int L, int d, int block,
                      int r, int out_dtype, unsigned flags, bool dense, void* stream_) {
  if (B <= 0 || H <= 0) return BB_ERR_INVALID_ARG;
  Layout lo;
  const int st = make_layout(L, d, block, r, flags, lo);
  if (st != BB_OK) return st;
  if (static_cast<int64_t>(B) * H * L >= (int64_t(1) << 31)) return BB_ERR_UNSUPPORTED;
  if (!q || !k || !lse || !out_rows) return BB_ERR_INVALID_ARG;
  if (!dense && lo.sparse && !out_band) return BB_ERR_INVALID_ARG;
  if (lo.sparse && !rand_attn) return BB_ERR_INVALID_ARG;
  if (out_dtype != BB_OUT_BF16 && out_dtype != BB_OUT_F32) return BB_ERR_INVALID_ARG;
  auto misaligned = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) != 0; };
  if (misaligned(q) || misaligned(k) || misaligned(out_rows) || (out_band && misaligned(out_band)))
    return BB_ERR_UNSUPPORTED;

  const int ranges = (lo.nb + kTiles - 1) / kTiles;
  const int chunks = lo.sparse ? (lo.band_slots + kTiles - 1) / kTiles : 0;
  const int64_t per_head =
      dense ? static_cast<int64_t>(lo.nb) * ranges : static_cast<int64_t>(lo.grows) * ranges +
                                                         static_cast<int64_t>(lo.band_rows) * chunks;
  const int64_t units = per_head * B * H;
  if (units >= (int64_t(1) << 31)) return BB_ERR_UNSUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BB_ERR_CUDA;
  uint32_t* status = status_word(dev);
  if (!status) return BB_ERR_UNSUPPORTED;

  CUtensorMap tq, tk;
  const uint64_t rows = static_cast<uint64_t>(B) * H * L;
  if (!make_tile_map(&tq, q, rows) || !make_tile_map(&tk, k, rows)) return BB_ERR_CUDA;

  ProbsParams p{};
  p.lse = lse;
  p.rand_attn = rand_attn;
  p.seq_mask = seq_mask;
  p.out_rows = out_rows;
  p.out_band = out_band;
  p.status = status;
  p.H = H;
  p.L = L;
  p.nb = lo.nb;
  p.r = r;
  p.sparse = lo.sparse ? 1 : 0;
  p.dense = dense ? 1 : 0;
  p.out_f32 = out_dtype == BB_OUT_F32 ? 1 : 0;
  p.ranges = ranges;
  p.chunks = chunks;
  p.grows = lo.grows;
  p.units_per_head = static_cast<int>(per_head);
  p.total_units = static_cast<int>(units);
  p.scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
  p.bias_log2 = -10000.0f * kLog2e;
  // Persistent grid: kCtasPerSm CTAs per SM at most, each taking an equal
  // run of consecutive units (neighbouring units share K tiles in L2).
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return BB_ERR_CUDA;
  const int64_t slots = static_cast<int64_t>(kCtasPerSm) * sms;
  p.units_per_cta = static_cast<int>((units + slots - 1) / slots);
  const int grid = static_cast<int>((units + p.units_per_cta - 1) / p.units_per_cta);

  const int smem = static_cast<int>(sizeof(Smem) + 1024);
  // (set on every call: the attribute is per device and the call is cheap)
  if (cudaFuncSetAttribute(bigbird_probs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return BB_ERR_CUDA;
  // Four CTAs (51 KB each) per SM need a large shared-memory carve-out.
  if (cudaFuncSetAttribute(bigbird_probs_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return BB_ERR_CUDA;
  bigbird_probs_kernel<<<grid, kThreads, smem, static_cast<cudaStream_t>(stream_)>>>(tq, tk, p);
  return cudaGetLastError() == cudaSuccess ? BB_OK : BB_ERR_CUDA;
}

}  // namespace bbp

extern "C" {

int bigbird_attn_probs_layout(int L, int d, int block, int r, unsigned flags, int* global_rows, int* band_rows,
                              int* band_slots) {
  bbp::Layout lo;
  const int st = bbp::make_layout(L, d, block, r, flags, lo);
  if (st != BB_OK) return st;
  if (global_rows) *global_rows = lo.grows;
  if (band_rows) *band_rows = lo.band_rows;
  if (band_slots) *band_slots = lo.band_slots;
  return BB_OK;
}

int bigbird_attn_probs(const void* q, const void* k, const float* lse, const int32_t* rand_attn,
                       const uint8_t* seq_mask, void* probs_global, void* probs_band, int B, int H, int L, int d,
                       int block, int r, int out_dtype, unsigned flags, void* stream) {
  return bbp::probs_impl(q, k, lse, rand_attn, seq_mask, probs_global, probs_band, B, H, L, d, block, r, out_dtype,
                         flags, false, stream);
}

int bigbird_attn_probs_dense(const void* q, const void* k, const float* lse, const int32_t* rand_attn,
                             const uint8_t* seq_mask, void* probs, int B, int H, int L, int d, int block, int r,
                             int out_dtype, unsigned flags, void* stream) {
  return bbp::probs_impl(q, k, lse, rand_attn, seq_mask, probs, nullptr, B, H, L, d, block, r, out_dtype, flags, true,
                         stream);
}

}  // extern "C"
