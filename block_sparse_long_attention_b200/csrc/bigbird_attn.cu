// BigBird ITC block-sparse attention forward for B200 (sm_100a).
//
// One persistent, warp-specialised kernel processes "units" of 128 query rows
// (two 64-row query blocks stacked, so every tensor-core MMA has M = 128):
//
//   * global units: query blocks 0 and nb-1 (or a pair of blocks in the
//     full-attention fallback) against a contiguous range of key blocks; with
//     more than one range per head the unit writes a partial (unnormalised
//     output, running max, running sum) that a small merge kernel combines by
//     log-sum-exp [TFG-BigBird, section "BigBird：从二次方注意力到线性稀疏注意力":
//     the first and last blocks attend to the whole K/V];
//   * pair units: query blocks i and i+1 (1 <= i <= nb-2) against the union of
//     their key blocks -- window, the two global blocks and their random blocks
//     rand_attn[h][i-1], rand_attn[h][i] -- with a per-block mask telling which
//     of the two 64-row halves uses the block [TFG-BigBird, same section and
//     "随机块掩码是如何生成的"; HF-Pegasus, section "三类注意力组合"]. A half that
//     does not use a block writes P = 0 for it, so the pair shares every MMA.
//
// Warp roles (192 threads): warps 0-3 run the softmax and the epilogue, one
// query row per thread (thread t owns TMEM lane t); warp 4 builds the unit's
// key-block list and key-validity masks and issues the TMA loads; warp 5
// allocates TMEM and issues the tcgen05 MMAs from one thread.
//
// Per key block j of a unit:  S_j = Q K_j^T        (SS MMA, 128x64x64, TMEM)
//                             P_j = exp2(S_j*c + bias - m)   (softmax warps, bf16
//                                   written back over S_j in TMEM)
//                             O  += P_j V_j        (TS MMA, P from TMEM)
// with an online softmax whose reference max is moved only when it grows by
// more than 2^8 (the O rescale is skipped otherwise; the final O / l is exact
// either way). Padded keys get -10000 added to the scaled score.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/bigbird_attn.h"
#include "sm100_ptx.cuh"

namespace bb {

constexpr int kBlock = 64;             // tokens per block
constexpr int kHeadDim = 64;           // head dimension
constexpr int kRows = 128;             // query rows per unit (two blocks)
constexpr int kStages = 4;             // K/V ring depth
constexpr int kMaxList = 40;           // key blocks per unit
constexpr int kMaxR = 16;              // random blocks per row supported
constexpr int kSplitBlocks = 8;        // key blocks per global-row range
constexpr int kThreads = 192;
constexpr uint32_t kTileBytes = kBlock * kHeadDim * 2;  // one 64x64 bf16 tile
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 128;        // O accumulator columns [128, 192)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kNegInit = -1.0e30f;

// status word bits
constexpr uint32_t kStatusBadRandAttn = 1u;
constexpr uint32_t kStatusTimeout = 2u;

__device__ uint32_t g_status;

struct UnitInfo {
  int32_t n;     // key blocks in the list
  int32_t bh;    // b * H + h
  int32_t qtop;  // query block of rows 0..63
  int32_t qbot;  // query block of rows 64..127, or -1
  int32_t split; // key range index of a partial global unit, or -1
  int32_t pad_;
  int32_t kb[kMaxList];
  uint64_t vm[kMaxList];  // bit c set: key c of the block is valid
  uint8_t hm[kMaxList];   // bit 0: rows 0..63 use the block, bit 1: rows 64..127
};

struct FwdParams {
  const int32_t* rand_attn;
  const uint8_t* seq_mask;
  void* out;
  float* part_o;   // [BH, nsplit, 128, 64]
  float* part_ml;  // [BH, nsplit, 128, 2]
  uint32_t* status;
  int B, H, L, nb, r, BH;
  int sparse;
  int nsplit;        // key ranges per global unit (1 = write the output directly)
  int split_blocks;  // key blocks per range
  int n_glob_units;
  int n_pairs;       // pair units per head
  int total_units;
  int out_f32;
  float scale_log2;  // log2(e) / sqrt(d)
  float bias_raw;    // -10000 * sqrt(d): the masked-key bias in units of q.k
};

struct __align__(1024) SharedStorage {
  uint8_t q[2][kRows * kHeadDim * 2];   // 2 x 16 KB, SW128, 1024-aligned
  uint8_t k[kStages][kTileBytes];       // 8 KB each
  uint8_t v[kStages][kTileBytes];
  UnitInfo unit[4];
  uint64_t q_full[2];
  uint64_t q_free[2];
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];
  uint64_t o_full;
  uint64_t o_free;
  uint32_t tmem_base;
  int32_t abort_flag;
};

__device__ __forceinline__ void flag_timeout(SharedStorage& s, const FwdParams& p) {
  atomicOr(p.status, kStatusTimeout);
  *reinterpret_cast<volatile int32_t*>(&s.abort_flag) = 1;
}

__device__ __forceinline__ bool aborted(SharedStorage& s) {
  return *reinterpret_cast<volatile int32_t*>(&s.abort_flag) != 0;
}

// Every lane waits (and acquires); the warp agrees on the outcome so that a
// timeout never splits the warp before a .sync.aligned instruction.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

// Decode unit u and build its key-block list. Called by a whole warp: the
// lanes fetch the unit's random entries in parallel, lane 0 builds the list.
__device__ void build_unit(const FwdParams& p, int u, UnitInfo& ui, int lane) {
  int n = 0;
  auto add = [&](int kb, int hm) {
    if (kb < 0 || kb >= p.nb) {
      atomicOr(p.status, kStatusBadRandAttn);
      return;
    }
    for (int e = 0; e < n; ++e)
      if (ui.kb[e] == kb) {
        ui.hm[e] |= static_cast<uint8_t>(hm);
        return;
      }
    ui.kb[n] = kb;
    ui.hm[n] = static_cast<uint8_t>(hm);
    ++n;
  };
  if (u < p.n_glob_units) {
    int bh, s, qtop, qbot;
    if (p.sparse) {
      bh = u / p.nsplit;
      s = u % p.nsplit;
      qtop = 0;
      qbot = p.nb - 1;
    } else {
      const int npair = (p.nb + 1) / 2;
      bh = u / (npair * p.nsplit);
      const int rem = u % (npair * p.nsplit);
      const int pp = rem / p.nsplit;
      s = rem % p.nsplit;
      qtop = 2 * pp;
      qbot = 2 * pp + 1 < p.nb ? 2 * pp + 1 : -1;
    }
    if (lane == 0) {
      const int k0 = s * p.split_blocks;
      const int k1 = min(p.nb, k0 + p.split_blocks);
      for (int kb = k0; kb < k1; ++kb) add(kb, 3);
      ui.bh = bh;
      ui.qtop = qtop;
      ui.qbot = qbot;
      ui.split = p.nsplit > 1 ? s : -1;
      ui.n = n;
    }
  } else {
    const int v = u - p.n_glob_units;
    const int bh = v / p.n_pairs;
    const int pp = v % p.n_pairs;
    const int qtop = 1 + 2 * pp;
    const int qbot = (2 + 2 * pp <= p.nb - 2) ? 2 + 2 * pp : -1;
    const int h = bh % p.H;
    const int both = qbot >= 0 ? 3 : 1;
    // rand_attn rows qtop-1 and qtop (= qbot-1) are adjacent: lane t < r reads
    // the top row's entry t, lane r + t the bottom row's entry t.
    const int nrand = qbot >= 0 ? 2 * p.r : p.r;
    const int32_t* ra = p.rand_attn + (static_cast<size_t>(h) * (p.nb - 2) + (qtop - 1)) * p.r;
    const int rv = lane < nrand ? __ldg(ra + lane) : -1;
    if (lane == 0) {
      add(qtop - 1, 1);
      add(qtop, both);
      add(qtop + 1, both);
      if (qbot >= 0) add(qtop + 2, 2);
      add(0, both);
      add(p.nb - 1, both);
    }
    for (int t = 0; t < nrand; ++t) {
      const int x = __shfl_sync(0xffffffffu, rv, t);
      if (lane == 0) add(x, t < p.r ? 1 : 2);
    }
    if (lane == 0) {
      ui.bh = bh;
      ui.qtop = qtop;
      ui.qbot = qbot;
      ui.split = -1;
      ui.n = n;
    }
  }
}

// 64 validity bits of key block kb of batch b (bit c: seq_mask of key c != 0).
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
__device__ void prep_unit(const FwdParams& p, int u, UnitInfo& ui, int lane) {
  build_unit(p, u, ui, lane);
  __syncwarp();
  const int n = ui.n;
  const int b = ui.bh / p.H;
  // Key validity bits: lane e handles list entries e and e + 32.
  for (int e = lane; e < n; e += 32)
    ui.vm[e] = p.seq_mask ? key_valid_bits(p.seq_mask, p.L, b, ui.kb[e]) : ~0ull;
  __syncwarp();
}

// The next unit's info is prepared while the current unit's first K/V tiles
// are in flight, so the list-building loads never stall the TMA ring at a
// unit boundary. Four info slots: a slot is rewritten three units after its
// last use, when every consumer is provably done with it.
__device__ void producer_role(SharedStorage& s, const FwdParams& p, const CUtensorMap* tmQ, const CUtensorMap* tmK,
                              const CUtensorMap* tmV) {
  const int lane = threadIdx.x & 31;
  const uint64_t pol_kv = l2_policy_evict_last();
  const uint64_t pol_q = l2_policy_evict_first();
  uint32_t unit_it = 0, kv_it = 0;
  int u = blockIdx.x;
  if (u < p.total_units) prep_unit(p, u, s.unit[0], lane);
  for (; u < p.total_units; u += gridDim.x, ++unit_it) {
    const int qs = unit_it & 1;
    const uint32_t ph = (unit_it >> 1) & 1;
    const UnitInfo& ui = s.unit[unit_it & 3];
    int ok = 1;
    if (lane == 0) ok = mbar_wait(smem_u32(&s.q_free[qs]), ph ^ 1);
    if (!__shfl_sync(0xffffffffu, ok, 0)) {
      if (lane == 0) flag_timeout(s, p);
      return;
    }
    const int n = ui.n;
    const int32_t row0 = ui.bh * p.L;
    const int nxt = u + gridDim.x;
    const int prep_at = min(n, kStages) - 1;
    if (lane == 0) {
      const uint32_t qbar = smem_u32(&s.q_full[qs]);
      mbar_arrive_expect_tx(qbar, ui.qbot >= 0 ? 2 * kTileBytes : kTileBytes);
      tma_load_2d(smem_u32(s.q[qs]), tmQ, qbar, 0, row0 + ui.qtop * kBlock, pol_q);
      if (ui.qbot >= 0) tma_load_2d(smem_u32(s.q[qs]) + kTileBytes, tmQ, qbar, 0, row0 + ui.qbot * kBlock, pol_q);
    }
    for (int j = 0; j < n; ++j, ++kv_it) {
      if (lane == 0) {
        const int st = kv_it % kStages;
        ok = mbar_wait(smem_u32(&s.kv_empty[st]), ((kv_it / kStages) & 1) ^ 1);
        if (ok) {
          const uint32_t kbar = smem_u32(&s.kv_full[st]);
          mbar_arrive_expect_tx(kbar, 2 * kTileBytes);
          const int32_t krow = row0 + ui.kb[j] * kBlock;
          tma_load_2d(smem_u32(s.k[st]), tmK, kbar, 0, krow, pol_kv);
          tma_load_2d(smem_u32(s.v[st]), tmV, kbar, 0, krow, pol_kv);
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) flag_timeout(s, p);
        return;
      }
      if (j == prep_at && nxt < p.total_units) prep_unit(p, nxt, s.unit[(unit_it + 1) & 3], lane);
    }
  }
}

// ---------------------------------------------------------------- MMA issuer

__device__ void mma_role(SharedStorage& s, const FwdParams& p, uint32_t tmem) {
  const uint32_t idesc_s = idesc_bf16_f32(kRows, kBlock, false);
  // P.V runs in fp16: P is written as fp16 and V is converted to fp16 in shared
  // memory (exact for bf16 values in the fp16 normal range); fp16 keeps three
  // more mantissa bits of P than bf16 would.
  const uint32_t idesc_o = idesc_f32acc(kRows, kHeadDim, false, true);
  uint32_t unit_it = 0, kv_it = 0, g = 0;
  bool ok = true;
  for (int u = blockIdx.x; u < p.total_units && ok; u += gridDim.x, ++unit_it) {
    const int slot = unit_it & 1;
    const uint32_t ph = (unit_it >> 1) & 1;
    if (!mbar_wait(smem_u32(&s.q_full[slot]), ph)) { ok = false; break; }
    const int n = s.unit[unit_it & 3].n;
    const uint32_t q_addr = smem_u32(s.q[slot]);

    auto issue_pv = [&](int jj) -> bool {
      const uint32_t gg = g + jj;
      const int sb = gg & 1;
      const int st = (kv_it + jj) % kStages;
      if (!mbar_wait(smem_u32(&s.p_full[sb]), (gg >> 1) & 1)) return false;
      if (jj == 0 && !mbar_wait(smem_u32(&s.o_free), (unit_it & 1) ^ 1)) return false;
      tc_fence_after();
      const uint32_t v_addr = smem_u32(s.v[st]);
#pragma unroll
      for (int kk = 0; kk < kBlock / 16; ++kk) {
        const uint64_t bdesc = sdesc_sw128(v_addr + kk * 2048, 8192, 1024);
        mma_ts(tmem + kColO, tmem + sb * 64 + kk * 8, bdesc, idesc_o, (jj > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(smem_u32(&s.pv_done[sb]));
      mma_commit(smem_u32(&s.kv_empty[st]));
      return true;
    };

    for (int j = 0; j < n && ok; ++j) {
      const uint32_t gg = g + j;
      const int sb = gg & 1;
      const uint32_t kvi = kv_it + j;
      const int st = kvi % kStages;
      if (!mbar_wait(smem_u32(&s.kv_full[st]), (kvi / kStages) & 1)) { ok = false; break; }
      if (gg >= 2 && !mbar_wait(smem_u32(&s.pv_done[sb]), ((gg >> 1) - 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t k_addr = smem_u32(s.k[st]);
#pragma unroll
      for (int kk = 0; kk < kHeadDim / 16; ++kk) {
        const uint64_t adesc = sdesc_sw128(q_addr + kk * 32, 16, 1024);
        const uint64_t bdesc = sdesc_sw128(k_addr + kk * 32, 16, 1024);
        mma_ss(tmem + sb * 64, adesc, bdesc, idesc_s, kk > 0 ? 1u : 0u);
      }
      mma_commit(smem_u32(&s.s_full[sb]));
      if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
    }
    if (!ok) break;
    if (n > 0 && !issue_pv(n - 1)) { ok = false; break; }
    mma_commit(smem_u32(&s.q_free[slot]));
    mma_commit(smem_u32(&s.o_full));
    kv_it += n;
    g += n;
  }
  if (!ok) flag_timeout(s, p);
}

// ---------------------------------------------------------------- softmax + epilogue

__device__ __forceinline__ float fmax_tree(const float (&x)[16]) {
  float a = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
  float b = fmaxf(fmaxf(x[4], x[5]), fmaxf(x[6], x[7]));
  float c = fmaxf(fmaxf(x[8], x[9]), fmaxf(x[10], x[11]));
  float d = fmaxf(fmaxf(x[12], x[13]), fmaxf(x[14], x[15]));
  return fmaxf(fmaxf(a, b), fmaxf(c, d));
}

__device__ void softmax_role(SharedStorage& s, const FwdParams& p, uint32_t tmem) {
  const int tid = threadIdx.x;  // 0..127 == TMEM lane
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int half = warp >> 1;   // 0: rows 0..63, 1: rows 64..127
  const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
  uint32_t unit_it = 0, g = 0;
  for (int u = blockIdx.x; u < p.total_units; u += gridDim.x, ++unit_it) {
    const int slot = unit_it & 1;
    const uint32_t ph = (unit_it >> 1) & 1;
    if (!warp_wait(smem_u32(&s.q_full[slot]), ph)) { flag_timeout(s, p); return; }
    const UnitInfo& ui = s.unit[unit_it & 3];
    const int n = ui.n;
    const int bh = ui.bh;
    const int qblk = half ? ui.qbot : ui.qtop;
    const int split = ui.split;
    const bool exists = qblk >= 0;
    float m_ref = kNegInit, l_run = 0.f;

    for (int j = 0; j < n; ++j) {
      const uint32_t gg = g + j;
      const int sb = gg & 1;
      if (!warp_wait(smem_u32(&s.s_full[sb]), (gg >> 1) & 1)) { flag_timeout(s, p); return; }
      tc_fence_after();
      const bool used = exists && ((ui.hm[j] >> half) & 1);
      uint32_t pk[32];
      if (used) {
        float x[64];  // raw scores q.k (+ the masked-key bias in the same units)
        {
          uint32_t r0[32], r1[32];
          tmem_ld32(tmem + lane_addr + sb * 64, r0);
          tmem_ld32(tmem + lane_addr + sb * 64 + 32, r1);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            x[c] = __uint_as_float(r0[c]);
            x[32 + c] = __uint_as_float(r1[c]);
          }
        }
        const uint64_t vm = ui.vm[j];
        if (vm != ~0ull) {
#pragma unroll
          for (int c = 0; c < 64; ++c) x[c] += ((vm >> c) & 1ull) ? 0.f : p.bias_raw;
        }
        float mx;
        {
          float t[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) t[c] = fmaxf(fmaxf(x[c], x[16 + c]), fmaxf(x[32 + c], x[48 + c]));
          mx = fmax_tree(t) * p.scale_log2;
        }
        float factor = 1.f;
        bool rescale_o = false;
        if (mx > m_ref + kRescaleThreshold) {
          factor = ex2_approx(m_ref - mx);
          rescale_o = l_run > 0.f;
          m_ref = mx;
        }
        const float neg_m = -m_ref;
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float e0 = ex2_approx(fmaf(x[2 * c], p.scale_log2, neg_m));
          const float e1 = ex2_approx(fmaf(x[2 * c + 1], p.scale_log2, neg_m));
          sum += e0 + e1;
          pk[c] = pack_f16x2(e0, e1);
        }
        l_run = l_run * factor + sum;
        if (__any_sync(0xffffffffu, rescale_o)) {
          // O rows are final only once the previous block's P.V has landed.
          const uint32_t gp = gg - 1;
          if (!warp_wait(smem_u32(&s.pv_done[gp & 1]), (gp >> 1) & 1)) { flag_timeout(s, p); return; }
          tc_fence_after();
#pragma unroll
          for (int c0 = 0; c0 < 64; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_addr + kColO + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * factor);
            tmem_st32(tmem + lane_addr + kColO + c0, o);
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      {
        // Convert this thread's 64-byte slice of V_j to fp16 in place (the
        // block counter is also the K/V ring counter).
        const int st = gg % kStages;
        if (!warp_wait(smem_u32(&s.kv_full[st]), (gg / kStages) & 1)) { flag_timeout(s, p); return; }
        uint4* vp = reinterpret_cast<uint4*>(s.v[st]) + tid * 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 w = vp[i];
          w.x = bf16x2_to_f16x2(w.x);
          w.y = bf16x2_to_f16x2(w.y);
          w.z = bf16x2_to_f16x2(w.z);
          w.w = bf16x2_to_f16x2(w.w);
          vp[i] = w;
        }
        fence_proxy_async_smem();
      }
      tmem_st32(tmem + lane_addr + sb * 64, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&s.p_full[sb]));
    }

    // ---- epilogue
    if (!warp_wait(smem_u32(&s.o_full), unit_it & 1)) { flag_timeout(s, p); return; }
    tc_fence_after();
    uint32_t o0[32], o1[32];
    tmem_ld32(tmem + lane_addr + kColO, o0);
    tmem_ld32(tmem + lane_addr + kColO + 32, o1);
    tmem_wait_ld();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(smem_u32(&s.o_free));
    }
    if (exists) {
      const int row_in_blk = tid & 63;
      if (split >= 0) {
        const size_t base = (static_cast<size_t>(bh) * p.nsplit + split) * kRows + tid;
        float4* dst = reinterpret_cast<float4*>(p.part_o + base * kHeadDim);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          dst[c] = make_float4(__uint_as_float(o0[4 * c]), __uint_as_float(o0[4 * c + 1]),
                               __uint_as_float(o0[4 * c + 2]), __uint_as_float(o0[4 * c + 3]));
#pragma unroll
        for (int c = 0; c < 8; ++c)
          dst[8 + c] = make_float4(__uint_as_float(o1[4 * c]), __uint_as_float(o1[4 * c + 1]),
                                   __uint_as_float(o1[4 * c + 2]), __uint_as_float(o1[4 * c + 3]));
        reinterpret_cast<float2*>(p.part_ml)[base] = make_float2(m_ref, l_run);
      } else {
        const float inv = 1.f / l_run;
        const size_t row = static_cast<size_t>(bh) * p.L + static_cast<size_t>(qblk) * kBlock + row_in_blk;
        if (p.out_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * kHeadDim);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            dst[c] = make_float4(__uint_as_float(o0[4 * c]) * inv, __uint_as_float(o0[4 * c + 1]) * inv,
                                 __uint_as_float(o0[4 * c + 2]) * inv, __uint_as_float(o0[4 * c + 3]) * inv);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            dst[8 + c] = make_float4(__uint_as_float(o1[4 * c]) * inv, __uint_as_float(o1[4 * c + 1]) * inv,
                                     __uint_as_float(o1[4 * c + 2]) * inv, __uint_as_float(o1[4 * c + 3]) * inv);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + row * kHeadDim);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            dst[c] = make_uint4(pack_bf16x2(__uint_as_float(o0[8 * c]) * inv, __uint_as_float(o0[8 * c + 1]) * inv),
                                pack_bf16x2(__uint_as_float(o0[8 * c + 2]) * inv, __uint_as_float(o0[8 * c + 3]) * inv),
                                pack_bf16x2(__uint_as_float(o0[8 * c + 4]) * inv, __uint_as_float(o0[8 * c + 5]) * inv),
                                pack_bf16x2(__uint_as_float(o0[8 * c + 6]) * inv, __uint_as_float(o0[8 * c + 7]) * inv));
#pragma unroll
          for (int c = 0; c < 4; ++c)
            dst[4 + c] = make_uint4(pack_bf16x2(__uint_as_float(o1[8 * c]) * inv, __uint_as_float(o1[8 * c + 1]) * inv),
                                    pack_bf16x2(__uint_as_float(o1[8 * c + 2]) * inv, __uint_as_float(o1[8 * c + 3]) * inv),
                                    pack_bf16x2(__uint_as_float(o1[8 * c + 4]) * inv, __uint_as_float(o1[8 * c + 5]) * inv),
                                    pack_bf16x2(__uint_as_float(o1[8 * c + 6]) * inv, __uint_as_float(o1[8 * c + 7]) * inv));
        }
      }
    }
    g += n;
  }
}

__global__ void __launch_bounds__(kThreads, 2)
bigbird_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  SharedStorage& s = *reinterpret_cast<SharedStorage*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (warp == 5) {
    tmem_alloc(smem_u32(&s.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s.q_full[i]), 1);
      mbar_init(smem_u32(&s.q_free[i]), 1);
      mbar_init(smem_u32(&s.s_full[i]), 1);
      mbar_init(smem_u32(&s.p_full[i]), 4);
      mbar_init(smem_u32(&s.pv_done[i]), 1);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&s.kv_full[i]), 1);
      mbar_init(smem_u32(&s.kv_empty[i]), 1);
    }
    mbar_init(smem_u32(&s.o_full), 1);
    mbar_init(smem_u32(&s.o_free), 4);
    s.abort_flag = 0;
    fence_barrier_init();
  }
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
    softmax_role(s, p, tmem);
  } else if (warp == 4) {
    producer_role(s, p, &tmQ, &tmK, &tmV);
  } else if (lane == 0) {
    mma_role(s, p, tmem);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Combine the partial results of the key ranges of the global rows by
// log-sum-exp (log2 units). 16 threads per query row, 4 columns each; a CTA
// covers 16 rows, grid = (B*H, 128 / 16).
constexpr int kMergeRowsPerCta = 16;

__global__ void __launch_bounds__(256)
bigbird_merge_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml, void* out, int nsplit,
                     int L, int nb, int out_f32) {
  const int bh = blockIdx.x;
  const int row = blockIdx.y * kMergeRowsPerCta + (threadIdx.x >> 4);
  const int c4 = threadIdx.x & 15;
  const size_t base = static_cast<size_t>(bh) * nsplit * kRows + row;
  const float2* ml = reinterpret_cast<const float2*>(part_ml);
  float mmax = kNegInit;
  for (int s = 0; s < nsplit; ++s) mmax = fmaxf(mmax, __ldg(&ml[base + static_cast<size_t>(s) * kRows].x));
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float l = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const size_t idx = base + static_cast<size_t>(s) * kRows;
    const float2 e = __ldg(&ml[idx]);
    const float w = ex2_approx(e.x - mmax);
    l += w * e.y;
    const float4 t = __ldg(reinterpret_cast<const float4*>(part_o + idx * kHeadDim) + c4);
    acc.x += w * t.x;
    acc.y += w * t.y;
    acc.z += w * t.z;
    acc.w += w * t.w;
  }
  const float inv = 1.f / l;
  const int qblk = row < kBlock ? 0 : nb - 1;
  const size_t orow = static_cast<size_t>(bh) * L + static_cast<size_t>(qblk) * kBlock + (row & (kBlock - 1));
  if (out_f32) {
    reinterpret_cast<float4*>(static_cast<float*>(out) + orow * kHeadDim)[c4] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  } else {
    reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + orow * kHeadDim)[c4] =
        make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
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
static bool make_map(CUtensorMap* map, const void* base, uint64_t rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kHeadDim) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kHeadDim), static_cast<cuuint32_t>(kBlock)};
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
      const int smem = static_cast<int>(sizeof(SharedStorage) + 1024);
      if (cudaFuncSetAttribute(bigbird_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return nullptr;
      if (cudaGetSymbolAddress(reinterpret_cast<void**>(&di.status), g_status) != cudaSuccess) return nullptr;
    }
    di.attr_set = true;
  }
  return &di;
}

struct Plan {
  int nb = 0;
  bool sparse = false;
  int nsplit = 1;
  int split_blocks = 0;
  size_t ws_bytes = 0;
};

static int make_plan(int B, int H, int L, int d, int block, int r, unsigned flags, Plan& pl) {
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0 || block <= 0 || r < 1 || L % block != 0) return BB_ERR_INVALID_ARG;
  if (d != kHeadDim || block != kBlock || r > kMaxR) return BB_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * L >= (int64_t(1) << 31)) return BB_ERR_UNSUPPORTED;
  pl.nb = L / block;
  pl.sparse = (flags & BB_FLAG_FORCE_SPARSE) || pl.nb > 5 + 2 * r;
  if (pl.sparse && pl.nb < 5 + r) return BB_ERR_INVALID_ARG;
  if (pl.sparse) {
    pl.split_blocks = kSplitBlocks;
    pl.nsplit = (pl.nb + kSplitBlocks - 1) / kSplitBlocks;
  } else {
    pl.split_blocks = pl.nb;  // nb <= 5 + 2r <= kMaxList
    pl.nsplit = 1;
  }
  if (pl.nsplit > 1)
    pl.ws_bytes = static_cast<size_t>(B) * H * pl.nsplit * kRows * (kHeadDim + 2) * sizeof(float);
  return BB_OK;
}

}  // namespace bb

using namespace bb;

extern "C" {

size_t bigbird_attn_workspace_size(int B, int H, int L, int d, int block, int r, unsigned flags) {
  Plan pl;
  if (make_plan(B, H, L, d, block, r, flags, pl) != BB_OK) return 0;
  return pl.ws_bytes;
}

int bigbird_attn_fwd_ex(const void* q, const void* k, const void* v, const int32_t* rand_attn,
                        const uint8_t* seq_mask, void* out, int B, int H, int L, int d, int block, int r,
                        int out_dtype, unsigned flags, void* workspace, size_t workspace_bytes, void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  Plan pl;
  int st = make_plan(B, H, L, d, block, r, flags, pl);
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
  if (!make_map(&tq, q, rows) || !make_map(&tk, k, rows) || !make_map(&tv, v, rows)) return BB_ERR_CUDA;

  FwdParams p{};
  p.rand_attn = rand_attn;
  p.seq_mask = seq_mask;
  p.out = out;
  p.B = B;
  p.H = H;
  p.L = L;
  p.nb = pl.nb;
  p.r = r;
  p.BH = B * H;
  p.sparse = pl.sparse ? 1 : 0;
  p.nsplit = pl.nsplit;
  p.split_blocks = pl.split_blocks;
  if (pl.sparse) {
    p.n_glob_units = p.BH * pl.nsplit;
    p.n_pairs = (pl.nb - 2 + 1) / 2;
    p.total_units = p.n_glob_units + p.BH * p.n_pairs;
  } else {
    p.n_glob_units = p.BH * ((pl.nb + 1) / 2);
    p.n_pairs = 0;
    p.total_units = p.n_glob_units;
  }
  p.out_f32 = out_dtype == BB_OUT_F32 ? 1 : 0;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(d));
  p.bias_raw = -10000.0f * sqrtf(static_cast<float>(d));

  p.status = di->status;

  void* ws = workspace;
  bool owned = false;
  if (pl.ws_bytes > 0 && !ws) {
    if (cudaMallocAsync(&ws, pl.ws_bytes, stream) != cudaSuccess) return BB_ERR_CUDA;
    owned = true;
  }
  if (pl.ws_bytes > 0) {
    p.part_o = static_cast<float*>(ws);
    p.part_ml = p.part_o + static_cast<size_t>(p.BH) * pl.nsplit * kRows * kHeadDim;
  }

  const int grid = std::min(p.total_units, 2 * di->sms);
  const size_t smem = sizeof(SharedStorage) + 1024;
  bigbird_fwd_kernel<<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && pl.nsplit > 1) {
    bigbird_merge_kernel<<<dim3(p.BH, kRows / kMergeRowsPerCta), 256, 0, stream>>>(p.part_o, p.part_ml, out, pl.nsplit,
                                                                               L, pl.nb, p.out_f32);
    e = cudaGetLastError();
  }
  if (owned) cudaFreeAsync(ws, stream);
  return e == cudaSuccess ? BB_OK : BB_ERR_CUDA;
}

int bigbird_attn_fwd(const void* q, const void* k, const void* v, const int32_t* rand_attn, const uint8_t* seq_mask,
                     void* out, int B, int H, int L, int d, int block, int r, void* stream) {
  return bigbird_attn_fwd_ex(q, k, v, rand_attn, seq_mask, out, B, H, L, d, block, r, BB_OUT_BF16, 0u, nullptr, 0,
                             stream);
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
