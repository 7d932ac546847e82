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
// any row with its unlisted tiles zero (dense). One CTA per unit, 288 threads:
//   warp 8     TMEM allocation, TMA loads of the Q block and the listed K
//              tiles, and the MMAs. Scores are computed transposed,
//              S^T = K Q^T, two key tiles at a time (M = 128 keys, N = 64
//              queries, four tcgen05 128x64x16 steps), into one of two
//              64-column TMEM buffers;
//   warps 0-7  thread (warp w, lane l) reads TMEM lane 32 (w % 4) + l (one
//              key) and the 32 query columns of half w / 4, and writes p for
//              them. Consecutive lanes hold consecutive keys, so each store
//              instruction of a warp covers 32 consecutive elements of one
//              output row (128 bytes in fp32) with no shuffle. Zero tiles are
//              written with 16-byte stores while the MMAs run.
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
constexpr int kThreads = kEpiThreads + 32;  // + the TMEM / TMA / MMA warp
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
  float scale_log2;    // log2(e) / sqrt(d)
  float bias_raw;      // -10000 * sqrt(d): the masked-key bias in units of q.k
};

struct __align__(1024) Smem {
  uint8_t q[kTileBytes];          // the unit's Q block (SW128)
  uint8_t k[kTiles][kTileBytes];  // listed K tiles in compute order; slots 2g, 2g+1 form one M = 128 operand
  float lse2[kBlock];             // lse * log2(e) of the block's 64 rows
  long long tile_off[kTiles];     // element offset of each tile's (0, 0) in its output
  int32_t tile_kb[kTiles];        // key block of each tile, or -1 for a zero tile
  int32_t comp_tile[kTiles];      // compute slot -> tile index
  uint64_t ld_full;
  uint64_t mma_done[2];
  uint64_t tmem_free[2];
  uint64_t mma_all;
  uint32_t tmem_base;
  int32_t n_tiles, n_comp, ld, bh, qblk, band;
  int32_t abort_flag;
};

// Sorted distinct key blocks of band row i (1 <= i <= nb-2) of head h: the
// two global blocks, the window and the row's random blocks. Out-of-range
// random entries are skipped and reported in the status word.
__device__ int band_list(const ProbsParams& p, int h, int i, int32_t* lst) {
  int n = 0;
  auto add = [&](int x) {
    int pos = 0;
    while (pos < n && lst[pos] < x) ++pos;
    if (pos < n && lst[pos] == x) return;
    for (int t = n; t > pos; --t) lst[t] = lst[t - 1];
    lst[pos] = x;
    ++n;
  };
  add(0);
  add(p.nb - 1);
  add(i - 1);
  add(i);
  add(i + 1);
  const int32_t* ra = p.rand_attn + (static_cast<long long>(h) * (p.nb - 2) + (i - 1)) * p.r;
  for (int t = 0; t < p.r; ++t) {
    const int x = ra[t];
    if (x < 0 || x >= p.nb) {
      atomicOr(p.status, kStatusBadRandAttn);
      continue;
    }
    add(x);
  }
  return n;
}

// Decode unit `unit` into its query block, tiles, output offsets (one thread).
__device__ void plan_unit(const ProbsParams& p, Smem& sm, int unit) {
  const int bh = unit / p.units_per_head;
  int w = unit - bh * p.units_per_head;
  const int h = bh % p.H;
  const long long L = p.L;
  int i = 0, n_tiles = 0, ld = p.L, band = 0;
  int32_t lst[5 + kMaxR];
  if (p.dense) {
    i = w / p.ranges;
    const int j = w - i * p.ranges;
    const bool full = !p.sparse || i == 0 || i == p.nb - 1;
    const int n = full ? 0 : band_list(p, h, i, lst);
    const int kb0 = j * kTiles;
    n_tiles = min(kTiles, p.nb - kb0);
    for (int t = 0; t < n_tiles; ++t) {
      const int kb = kb0 + t;
      bool listed = full;
      for (int e = 0; e < n && !listed; ++e) listed = lst[e] == kb;
      sm.tile_kb[t] = listed ? kb : -1;
      sm.tile_off[t] = (static_cast<long long>(bh) * L + static_cast<long long>(i) * kBlock) * L +
                       static_cast<long long>(kb) * kBlock;
    }
  } else if (w < p.grows * p.ranges) {
    const int g = w / p.ranges;
    const int j = w - g * p.ranges;
    i = p.sparse ? (g == 0 ? 0 : p.nb - 1) : g;
    const int kb0 = j * kTiles;
    n_tiles = min(kTiles, p.nb - kb0);
    for (int t = 0; t < n_tiles; ++t) {
      const int kb = kb0 + t;
      sm.tile_kb[t] = kb;
      sm.tile_off[t] = (static_cast<long long>(bh) * p.grows + g) * kBlock * L + static_cast<long long>(kb) * kBlock;
    }
  } else {
    w -= p.grows * p.ranges;
    i = 1 + w / p.chunks;
    const int c = w - (i - 1) * p.chunks;
    const int slots = 5 + p.r;
    const int n = band_list(p, h, i, lst);
    const int s0 = c * kTiles;
    n_tiles = min(kTiles, slots - s0);
    ld = kBlock;
    band = 1;
    for (int t = 0; t < n_tiles; ++t) {
      const int s = s0 + t;
      sm.tile_kb[t] = s < n ? lst[s] : -1;
      sm.tile_off[t] =
          ((static_cast<long long>(bh) * (p.nb - 2) + (i - 1)) * slots + s) * static_cast<long long>(kBlock * kBlock);
    }
  }
  int nc = 0;
  for (int t = 0; t < n_tiles; ++t)
    if (sm.tile_kb[t] >= 0) sm.comp_tile[nc++] = t;
  sm.n_tiles = n_tiles;
  sm.n_comp = nc;
  sm.ld = ld;
  sm.bh = bh;
  sm.qblk = i;
  sm.band = band;
}

__device__ __forceinline__ void epi_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kEpiThreads) : "memory");
}

__global__ void __launch_bounds__(kThreads, 3)
bigbird_probs_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const ProbsParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (warp == kEpiWarps) {
    if (lane == 0) {
      mbar_init(smem_u32(&sm.ld_full), 1);
      for (int b = 0; b < 2; ++b) {
        mbar_init(smem_u32(&sm.mma_done[b]), 1);
        mbar_init(smem_u32(&sm.tmem_free[b]), kEpiThreads);
      }
      mbar_init(smem_u32(&sm.mma_all), 1);
      fence_barrier_init();
      sm.abort_flag = 0;
      plan_unit(p, sm, blockIdx.x);
    }
    __syncwarp();
    tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int nc = sm.n_comp;
  const int ngroups = (nc + 1) / 2;
  uint8_t* out = static_cast<uint8_t*>(sm.band ? p.out_band : p.out_rows);
  const int esize = p.out_f32 ? 4 : 2;

  if (warp == kEpiWarps) {
    // ---------------------------------------------------------------- TMA + MMA
    if (lane == 0 && nc > 0) {  // (a unit of zero tiles only loads nothing)
      const uint32_t full = smem_u32(&sm.ld_full);
      const uint64_t keep = l2_policy_evict_last();
      const int row0 = sm.bh * p.L;
      mbar_arrive_expect_tx(full, static_cast<uint32_t>(1 + nc) * kTileBytes);
      tma_load_2d(smem_u32(sm.q), &tmQ, full, 0, row0 + sm.qblk * kBlock, keep);
      for (int s = 0; s < nc; ++s)
        tma_load_2d(smem_u32(sm.k[s]), &tmK, full, 0, row0 + sm.tile_kb[sm.comp_tile[s]] * kBlock, keep);
      int issued = 0;
      if (!mbar_wait(full, 0)) {
        atomicOr(p.status, kStatusTimeout);
        *reinterpret_cast<volatile int32_t*>(&sm.abort_flag) = 1;
        mbar_arrive(smem_u32(&sm.mma_done[0]));
        mbar_arrive(smem_u32(&sm.mma_done[1]));
      } else {
        tc_fence_after();
        const uint32_t idesc = idesc_f32acc(2 * kBlock, kBlock, true, false);  // bf16 K . Q^T, M = 128, N = 64
        const uint32_t qa = smem_u32(sm.q);
        for (int g = 0; g < ngroups; ++g) {
          const int buf = g & 1;
          if (g >= 2 && !mbar_wait(smem_u32(&sm.tmem_free[buf]), ((g - 2) >> 1) & 1)) {
            atomicOr(p.status, kStatusTimeout);
            *reinterpret_cast<volatile int32_t*>(&sm.abort_flag) = 1;
            mbar_arrive(smem_u32(&sm.mma_done[buf]));
            break;
          }
          tc_fence_after();
          const uint32_t ka = smem_u32(sm.k[2 * g]);
#pragma unroll
          for (int kk = 0; kk < kDim / 16; ++kk)
            mma_ss(tmem + static_cast<uint32_t>(buf) * kBlock, sdesc_sw128(ka + kk * 32, 16, 1024),
                   sdesc_sw128(qa + kk * 32, 16, 1024), idesc, kk > 0 ? 1u : 0u);
          mma_commit(smem_u32(&sm.mma_done[buf]));
          issued = 1;
        }
      }
      if (issued) mma_commit(smem_u32(&sm.mma_all));
      // Before TMEM is released: every MMA has completed, and no copy is left
      // in flight (both bounded; only an earlier failure makes them wait).
      if (issued && !mbar_wait(smem_u32(&sm.mma_all), 0)) atomicOr(p.status, kStatusTimeout);
      if (!mbar_wait(full, 0)) atomicOr(p.status, kStatusTimeout);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- weights
    const int et = tid;  // 0 .. 255
    if (et < kBlock)
      sm.lse2[et] = p.lse[static_cast<long long>(sm.bh) * p.L + sm.qblk * kBlock + et] * kLog2e;
    // Zero tiles, while the loads and MMAs run.
    const int vec_per_row = kBlock * esize / 16;
    for (int t = 0; t < sm.n_tiles; ++t) {
      if (sm.tile_kb[t] >= 0) continue;
      uint8_t* base = out + sm.tile_off[t] * esize;
      for (int idx = et; idx < kBlock * vec_per_row; idx += kEpiThreads) {
        const int row = idx / vec_per_row;
        const int col = idx - row * vec_per_row;
        __stcs(reinterpret_cast<uint4*>(base + (static_cast<long long>(row) * sm.ld) * esize) + col,
               make_uint4(0u, 0u, 0u, 0u));
      }
    }
    epi_bar_sync();  // lse2 visible to every weight thread

    const int quad = warp & 3;                 // TMEM lanes 32 quad .. 32 quad + 31
    const int half = warp >> 2;                // query columns 32 half .. 32 half + 31
    const int m = 32 * quad + lane;            // key row of the 128-key pair
    const int b = sm.bh / p.H;
    const long long ld = sm.ld;
    for (int g = 0; g < ngroups; ++g) {
      const int buf = g & 1;
      const bool ok = mbar_wait(smem_u32(&sm.mma_done[buf]), (g >> 1) & 1);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) atomicOr(p.status, kStatusTimeout);
        *reinterpret_cast<volatile int32_t*>(&sm.abort_flag) = 1;
        break;
      }
      if (__any_sync(0xffffffffu, *reinterpret_cast<volatile int32_t*>(&sm.abort_flag) != 0)) break;
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * quad) << 16) + static_cast<uint32_t>(buf * kBlock + 32 * half), v);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.tmem_free[buf]));
      const int cs = 2 * g + (m >> 6);
      if (cs < nc) {
        const int ti = sm.comp_tile[cs];
        const int kb = sm.tile_kb[ti];
        const int kk = m & (kBlock - 1);
        const bool masked = p.seq_mask && !p.seq_mask[static_cast<long long>(b) * p.L + kb * kBlock + kk];
        const float braw = masked ? p.bias_raw : 0.0f;
        const long long base = sm.tile_off[ti] + kk + static_cast<long long>(32 * half) * ld;
        if (p.out_f32) {
          float* o = reinterpret_cast<float*>(out) + base;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float x = fmaf(__uint_as_float(v[c]) + braw, p.scale_log2, -sm.lse2[32 * half + c]);
            __stcs(o + c * ld, ex2_approx(x));
          }
        } else {
          unsigned short* o = reinterpret_cast<unsigned short*>(out) + base;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float x = fmaf(__uint_as_float(v[c]) + braw, p.scale_log2, -sm.lse2[32 * half + c]);
            __stcs(o + c * ld, __bfloat16_as_ushort(__float2bfloat16_rn(ex2_approx(x))));
          }
        }
      }
    }
  }

  __syncthreads();
  if (warp == kEpiWarps) {
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
  p.scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
  p.bias_raw = -10000.0f * sqrtf(static_cast<float>(d));

  const int smem = static_cast<int>(sizeof(Smem) + 1024);
  // (set on every call: the attribute is per device and the call is cheap)
  if (cudaFuncSetAttribute(bigbird_probs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return BB_ERR_CUDA;
  // Three CTAs (74 KB each) per SM need the largest shared-memory carve-out.
  if (cudaFuncSetAttribute(bigbird_probs_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return BB_ERR_CUDA;
  bigbird_probs_kernel<<<static_cast<unsigned>(units), kThreads, smem, static_cast<cudaStream_t>(stream_)>>>(tq, tk,
                                                                                                            p);
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
