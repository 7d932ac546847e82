// BigBird ITC block-sparse attention forward on CUDA cores, for the block
// sizes and head dims the tensor-core kernel does not take: block 32 or 128,
// d 64 or 128 (block_size is the method's one size knob [HF-Pegasus, section
// "使用限制与注意事项"]). Same definition as the tensor-core path: query blocks
// 0 and nb-1 attend to every key, every other query block i to key blocks
// {0, nb-1, i-1, i, i+1} and its random blocks (a set: repeats add nothing)
// [TFG-BigBird, section "BigBird：从二次方注意力到线性稀疏注意力"; HF-Pegasus,
// section "三类注意力组合"], scores q.k / sqrt(d) with -10000 added for padded
// keys, full attention when nb <= 5 + 2r [HF-Pegasus, section
// "序列过短时的自动回退"].
//
// One CTA of 256 threads per (b, h, query block). TPR = 256 / block threads
// share a query row, each holding d / TPR of its (pre-scaled) q and of its
// output in registers. Key blocks are visited 32 keys at a time: the chunk's
// K and V are staged in shared memory as fp32, each thread forms its partial
// dot products with the chunk's keys, the TPR partners add them with
// shuffles, and the row's online softmax (one rescale per chunk, exp2 with
// the scale folded into q) accumulates p * v into the output slice. fp32
// arithmetic throughout; no tensor cores.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>

#include "../../include/bigbird_attn.h"
#include "bb_internal.h"

namespace bbg {

constexpr int kThreads = 256;
constexpr int kChunk = 32;  // keys staged per step
constexpr int kMaxR = 16;
constexpr uint32_t kStatusBadRandAttn = 1u;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.69314718055994531f;

struct GenParams {
  const uint16_t* q;  // bf16 [B, H, L, D]
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* rand_attn;  // [H, nb-2, r]
  const uint8_t* seq_mask;   // [B, L] or null
  void* out;                 // [B, H, L, D], bf16 or fp32
  float* lse;                // [B, H, L] natural-log log-sum-exp, or null
  uint32_t* status;
  int H, L, nb, r;
  int sparse;
  int out_f32;
  float qscale;  // log2(e) / sqrt(D)
  float bias2;   // -10000 * log2(e)
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4 w, float* f) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = __uint_as_float(ws[j] << 16);
    f[2 * j + 1] = __uint_as_float(ws[j] & 0xFFFF0000u);
  }
}

template <int BS, int D>
__global__ void __launch_bounds__(kThreads) bigbird_generic_fwd_kernel(const GenParams p) {
  constexpr int TPR = kThreads / BS;  // threads per query row: 8 (block 32) or 2 (block 128)
  constexpr int SL = D / TPR;         // dims per thread: 8 .. 64, a multiple of 8
  static_assert(BS * TPR == kThreads && SL % 8 == 0 && BS % kChunk == 0, "tile shape");
  __shared__ __align__(16) float ks[kChunk][D];
  __shared__ __align__(16) float vs[kChunk][D];
  __shared__ float kbias[kChunk];
  __shared__ int32_t lst[5 + kMaxR];
  __shared__ int32_t nlst;

  const int i = blockIdx.x;  // query block
  const int bh = blockIdx.y;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int tid = threadIdx.x;
  const int row = tid / TPR;
  const int part = tid - row * TPR;
  const long long base = static_cast<long long>(bh) * p.L * D;
  const int qrow = i * BS + row;
  const bool full = !p.sparse || i == 0 || i == p.nb - 1;

  if (tid == 0 && !full) {
    // sorted distinct key blocks of row i; out-of-range random entries are skipped and flagged
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
    nlst = n;
  }

  float qv[SL];
  {
    const uint4* src = reinterpret_cast<const uint4*>(p.q + base + static_cast<long long>(qrow) * D + part * SL);
#pragma unroll
    for (int c = 0; c < SL / 8; ++c) {
      bf16x8_to_f32(src[c], qv + 8 * c);
#pragma unroll
      for (int e = 0; e < 8; ++e) qv[8 * c + e] *= p.qscale;
    }
  }
  float o[SL];
#pragma unroll
  for (int e = 0; e < SL; ++e) o[e] = 0.0f;
  float m = -1.0e30f, l = 0.0f;
  __syncthreads();
  const int nblk = full ? p.nb : nlst;

  for (int e = 0; e < nblk; ++e) {
    const int kb = full ? e : lst[e];
    for (int c0 = 0; c0 < BS; c0 += kChunk) {
      const int key0 = kb * BS + c0;
      __syncthreads();  // every thread is done with the previous chunk
      for (int idx = tid; idx < kChunk * D / 8; idx += kThreads) {
        const int kr = idx / (D / 8);
        const int kc = (idx - kr * (D / 8)) * 8;
        const long long g = base + static_cast<long long>(key0 + kr) * D + kc;
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(p.k + g), &ks[kr][kc]);
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(p.v + g), &vs[kr][kc]);
      }
      if (tid < kChunk)
        kbias[tid] = (p.seq_mask && !p.seq_mask[static_cast<long long>(b) * p.L + key0 + tid]) ? p.bias2 : 0.0f;
      __syncthreads();
      float s[kChunk];
      float cm = m;
#pragma unroll
      for (int kk = 0; kk < kChunk; ++kk) {
        float acc = 0.0f;
#pragma unroll
        for (int d4 = 0; d4 < SL; d4 += 4) {
          const float4 kv = *reinterpret_cast<const float4*>(&ks[kk][part * SL + d4]);
          acc = fmaf(qv[d4], kv.x, acc);
          acc = fmaf(qv[d4 + 1], kv.y, acc);
          acc = fmaf(qv[d4 + 2], kv.z, acc);
          acc = fmaf(qv[d4 + 3], kv.w, acc);
        }
#pragma unroll
        for (int off = TPR / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        s[kk] = acc + kbias[kk];
        cm = fmaxf(cm, s[kk]);
      }
      const float corr = exp2f(m - cm);
      l *= corr;
#pragma unroll
      for (int d0 = 0; d0 < SL; ++d0) o[d0] *= corr;
#pragma unroll
      for (int kk = 0; kk < kChunk; ++kk) {
        const float pk = exp2f(s[kk] - cm);
        l += pk;
#pragma unroll
        for (int d4 = 0; d4 < SL; d4 += 4) {
          const float4 vv = *reinterpret_cast<const float4*>(&vs[kk][part * SL + d4]);
          o[d4] = fmaf(pk, vv.x, o[d4]);
          o[d4 + 1] = fmaf(pk, vv.y, o[d4 + 1]);
          o[d4 + 2] = fmaf(pk, vv.z, o[d4 + 2]);
          o[d4 + 3] = fmaf(pk, vv.w, o[d4 + 3]);
        }
      }
      m = cm;
    }
  }

  const float inv = 1.0f / l;
  const long long off = base + static_cast<long long>(qrow) * D + part * SL;
  if (p.out_f32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + off);
#pragma unroll
    for (int c = 0; c < SL / 4; ++c)
      dst[c] = make_float4(o[4 * c] * inv, o[4 * c + 1] * inv, o[4 * c + 2] * inv, o[4 * c + 3] * inv);
  } else {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + off);
#pragma unroll
    for (int c = 0; c < SL / 8; ++c) {
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 t = __floats2bfloat162_rn(o[8 * c + 2 * j] * inv, o[8 * c + 2 * j + 1] * inv);
        w[j] = *reinterpret_cast<const uint32_t*>(&t);
      }
      dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  if (p.lse && part == 0) p.lse[static_cast<long long>(bh) * p.L + qrow] = (m + log2f(l)) * kLn2;
}

template <int BS, int D>
static int launch(const GenParams& p, int nb, int BH, cudaStream_t stream) {
  bigbird_generic_fwd_kernel<BS, D><<<dim3(nb, BH), kThreads, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? BB_OK : BB_ERR_CUDA;
}

}  // namespace bbg

namespace bb {

bool generic_fwd_supported(int d, int block) {
  return (d == 64 || d == 128) && (block == 32 || block == 64 || block == 128) && !(d == 64 && block == 64);
}

int generic_fwd(const void* q, const void* k, const void* v, const int32_t* rand_attn, const uint8_t* seq_mask,
                void* out, float* lse, int B, int H, int L, int d, int block, int r, int out_dtype, unsigned flags,
                void* stream_) {
  using namespace bbg;
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0 || block <= 0 || r < 1 || L % block != 0) return BB_ERR_INVALID_ARG;
  if (!generic_fwd_supported(d, block) || r > kMaxR) return BB_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * L >= (int64_t(1) << 31) || L / block > 65535 || B * H > 65535)
    return BB_ERR_UNSUPPORTED;
  const int nb = L / block;
  const bool sparse = (flags & BB_FLAG_FORCE_SPARSE) || nb > 5 + 2 * r;
  if (sparse && nb < 5 + r) return BB_ERR_INVALID_ARG;
  if (!q || !k || !v || !out) return BB_ERR_INVALID_ARG;
  if (sparse && !rand_attn) return BB_ERR_INVALID_ARG;
  if (out_dtype != BB_OUT_BF16 && out_dtype != BB_OUT_F32) return BB_ERR_INVALID_ARG;
  auto misaligned = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) != 0; };
  if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(out)) return BB_ERR_UNSUPPORTED;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (sparse && (flags & BB_FLAG_DEBUG_CHECKS)) {
    const size_t n = static_cast<size_t>(H) * (nb - 2) * r;
    int32_t* hbuf = static_cast<int32_t*>(malloc(n * sizeof(int32_t)));
    if (!hbuf) return BB_ERR_CUDA;
    cudaError_t e = cudaMemcpyAsync(hbuf, rand_attn, n * sizeof(int32_t), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    const int vs = e == cudaSuccess ? bigbird_rand_attn_validate(hbuf, H, L, block, r, 0) : BB_ERR_CUDA;
    free(hbuf);
    if (vs != BB_OK) return vs;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BB_ERR_CUDA;
  uint32_t* status = status_word(dev);
  if (!status) return BB_ERR_UNSUPPORTED;
  GenParams p{};
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.rand_attn = rand_attn;
  p.seq_mask = seq_mask;
  p.out = out;
  p.lse = lse;
  p.status = status;
  p.H = H;
  p.L = L;
  p.nb = nb;
  p.r = r;
  p.sparse = sparse ? 1 : 0;
  p.out_f32 = out_dtype == BB_OUT_F32 ? 1 : 0;
  p.qscale = kLog2e / sqrtf(static_cast<float>(d));
  p.bias2 = -10000.0f * kLog2e;
  const int BH = B * H;
  if (block == 32 && d == 64) return launch<32, 64>(p, nb, BH, stream);
  if (block == 128 && d == 64) return launch<128, 64>(p, nb, BH, stream);
  if (block == 32 && d == 128) return launch<32, 128>(p, nb, BH, stream);
  if (block == 64 && d == 128) return launch<64, 128>(p, nb, BH, stream);
  return launch<128, 128>(p, nb, BH, stream);
}

}  // namespace bb
