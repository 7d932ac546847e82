// Backward pass of BigBird ITC block-sparse attention for B200 (sm_100a).
//
// Gradients of sum(dout * out) with respect to q, k and v for the same block
// pattern as the forward [TFG-BigBird, section "BigBird：从二次方注意力到线性稀疏注意力";
// HF-Pegasus, section "三类注意力组合"], by the chain rule through each row's
// softmax: with p = exp(s - lse) recomputed from the forward's row
// log-sum-exp, D = rowsum(dout * out),
//   dv_k += p^T dout,  dp = dout v^T,  ds = p (dp - D),
//   dq   += ds k / sqrt(d),  dk_k += ds^T q / sqrt(d).
//
// One CTA per (b, h, query block i), 256 threads, fp32 CUDA-core arithmetic
// on 64x64 tiles staged in shared memory: the CTA walks the key blocks of row
// i (all of them for the global rows and the full-attention fallback; else
// the set {0, nb-1, i-1, i, i+1} and the row's random blocks), keeps dq_i in
// registers and adds its dk_j, dv_j contributions with fp32 atomics (a key
// block receives from every query block that attends to it).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/bigbird_attn.h"

namespace bbw {

constexpr int kBlock = 64;
constexpr int kDim = 64;
constexpr int kThreads = 256;
constexpr int kLd = kDim + 1;  // padded row stride of the fp32 tiles
constexpr int kMaxList = 5 + 16;

struct BwdParams {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const void* out;
  const uint16_t* dout;
  const float* lse;
  const int32_t* rand_attn;
  const uint8_t* seq_mask;
  float* dq;
  float* dk;
  float* dv;
  int H, L, nb, r;
  int sparse;
  int out_f32;
  float scale;  // 1 / sqrt(d)
};

struct Smem {
  float q[kBlock][kLd];
  float dout[kBlock][kLd];
  float k[kBlock][kLd];
  float v[kBlock][kLd];
  float p[kBlock][kLd];
  float ds[kBlock][kLd];
  float lse[kBlock];
  float dsum[kBlock];   // D = rowsum(dout * out)
  float bias[kBlock];   // 0 or -10000 per key of the current block
  int list[kMaxList];
  int nlist;
};

__device__ __forceinline__ float bf16_to_f32(uint16_t x) { return __uint_as_float(static_cast<uint32_t>(x) << 16); }

// A 64x64 bf16 tile (rows row0.., 64 values each) into fp32 shared memory.
__device__ __forceinline__ void load_tile(float (&dst)[kBlock][kLd], const uint16_t* src, size_t row0) {
  for (int e = threadIdx.x; e < kBlock * kDim / 2; e += kThreads) {
    const int rr = e / (kDim / 2);
    const int cc = 2 * (e % (kDim / 2));
    const uint32_t w = reinterpret_cast<const uint32_t*>(src + (row0 + rr) * kDim)[cc / 2];
    dst[rr][cc] = bf16_to_f32(static_cast<uint16_t>(w & 0xFFFFu));
    dst[rr][cc + 1] = bf16_to_f32(static_cast<uint16_t>(w >> 16));
  }
}

__global__ void __launch_bounds__(kThreads, 2) bigbird_bwd_kernel(const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(smem_raw);
  const int i = blockIdx.x;   // query block
  const int bh = blockIdx.y;  // b * H + h
  const int b = bh / p.H;
  const int h = bh % p.H;
  const int t = threadIdx.x;
  const int row = t >> 2;          // query row (S/dq phases) or key (dk/dv phase) of this thread
  const int c0 = (t & 3) * 16;     // its 16 columns
  const size_t head = static_cast<size_t>(bh) * p.L;
  const size_t q0 = head + static_cast<size_t>(i) * kBlock;

  // ---- row data: q, dout, lse and D = rowsum(dout * out)
  load_tile(s.q, p.q, q0);
  load_tile(s.dout, p.dout, q0);
  if (t < kBlock) s.lse[t] = p.lse[q0 + t];
  {
    // D of row `row`: four threads per row, 16 columns each, combined by shuffles.
    float acc = 0.f;
    const size_t o = (q0 + row) * kDim + c0;
    for (int x = 0; x < 16; ++x) {
      const float ov = p.out_f32 ? static_cast<const float*>(p.out)[o + x]
                                 : bf16_to_f32(static_cast<const uint16_t*>(p.out)[o + x]);
      acc += ov * bf16_to_f32(p.dout[o + x]);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if ((t & 3) == 0) s.dsum[row] = acc;
  }
  // ---- the row's key blocks
  const bool all = !p.sparse || i == 0 || i == p.nb - 1;
  if (t == 0 && !all) {
    int n = 0;
    auto add = [&](int kb) {
      if (kb < 0 || kb >= p.nb) return;  // out of range: skipped (the forward flags it)
      for (int e = 0; e < n; ++e)
        if (s.list[e] == kb) return;
      s.list[n++] = kb;
    };
    add(i - 1);
    add(i);
    add(i + 1);
    add(0);
    add(p.nb - 1);
    const int32_t* ra = p.rand_attn + (static_cast<size_t>(h) * (p.nb - 2) + (i - 1)) * p.r;
    for (int e = 0; e < p.r; ++e) add(ra[e]);
    s.nlist = n;
  }
  __syncthreads();
  const int nkb = all ? p.nb : s.nlist;
  const float log2e = 1.4426950408889634f;

  float dq[16];
#pragma unroll
  for (int x = 0; x < 16; ++x) dq[x] = 0.f;

  for (int e = 0; e < nkb; ++e) {
    const int j = all ? e : s.list[e];
    const size_t k0 = head + static_cast<size_t>(j) * kBlock;
    load_tile(s.k, p.k, k0);
    load_tile(s.v, p.v, k0);
    if (t < kBlock) s.bias[t] = (p.seq_mask && !p.seq_mask[static_cast<size_t>(b) * p.L + j * kBlock + t]) ? -10000.f : 0.f;
    __syncthreads();
    // p and ds of row `row`, keys c0..c0+15
    {
      const float lse2 = s.lse[row] * log2e;
      const float dr = s.dsum[row];
#pragma unroll 4
      for (int c = c0; c < c0 + 16; ++c) {
        float sc = 0.f, dp = 0.f;
#pragma unroll 16
        for (int x = 0; x < kDim; ++x) {
          sc = fmaf(s.q[row][x], s.k[c][x], sc);
          dp = fmaf(s.dout[row][x], s.v[c][x], dp);
        }
        const float pv = exp2f(fmaf(sc, p.scale, s.bias[c]) * log2e - lse2);
        s.p[row][c] = pv;
        s.ds[row][c] = pv * (dp - dr);
      }
    }
    __syncthreads();
    // dq of row `row`, columns c0..c0+15: sum over the block's keys
#pragma unroll 4
    for (int c = 0; c < kBlock; ++c) {
      const float w = s.ds[row][c];
#pragma unroll
      for (int x = 0; x < 16; ++x) dq[x] = fmaf(w, s.k[c][c0 + x], dq[x]);
    }
    // dk and dv of key `row` of block j, columns c0..c0+15: sum over the query rows
    {
      float dk[16], dv[16];
#pragma unroll
      for (int x = 0; x < 16; ++x) dk[x] = dv[x] = 0.f;
#pragma unroll 4
      for (int rr = 0; rr < kBlock; ++rr) {
        const float w = s.ds[rr][row];
        const float pw = s.p[rr][row];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          dk[x] = fmaf(w, s.q[rr][c0 + x], dk[x]);
          dv[x] = fmaf(pw, s.dout[rr][c0 + x], dv[x]);
        }
      }
      float* dkp = p.dk + (k0 + row) * kDim + c0;
      float* dvp = p.dv + (k0 + row) * kDim + c0;
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        atomicAdd(dkp + x, dk[x] * p.scale);
        atomicAdd(dvp + x, dv[x]);
      }
    }
    __syncthreads();
  }
  float* dqp = p.dq + (q0 + row) * kDim + c0;
#pragma unroll
  for (int x = 0; x < 16; ++x) dqp[x] = dq[x] * p.scale;
}

}  // namespace bbw

extern "C" int bigbird_attn_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
                                const float* lse, const int32_t* rand_attn, const uint8_t* seq_mask, float* dq,
                                float* dk, float* dv, int B, int H, int L, int d, int block, int r, int out_dtype,
                                unsigned flags, void* stream_) {
  using namespace bbw;
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0 || block <= 0 || r < 1 || L % block != 0) return BB_ERR_INVALID_ARG;
  if (d != kDim || block != kBlock || r > 16) return BB_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * L >= (int64_t(1) << 31)) return BB_ERR_UNSUPPORTED;
  if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv) return BB_ERR_INVALID_ARG;
  if (out_dtype != BB_OUT_BF16 && out_dtype != BB_OUT_F32) return BB_ERR_INVALID_ARG;
  const int nb = L / block;
  const bool sparse = (flags & BB_FLAG_FORCE_SPARSE) || nb > 5 + 2 * r;
  if (sparse && nb < 5 + r) return BB_ERR_INVALID_ARG;
  if (sparse && !rand_attn) return BB_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  const size_t bytes = static_cast<size_t>(B) * H * L * d * sizeof(float);
  if (cudaMemsetAsync(dk, 0, bytes, stream) != cudaSuccess) return BB_ERR_CUDA;
  if (cudaMemsetAsync(dv, 0, bytes, stream) != cudaSuccess) return BB_ERR_CUDA;
  // (set on every call: the attribute is per device and the call is cheap)
  const int smem = static_cast<int>(sizeof(Smem));
  if (cudaFuncSetAttribute(bigbird_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return BB_ERR_CUDA;
  BwdParams p{};
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.out = out;
  p.dout = static_cast<const uint16_t*>(dout);
  p.lse = lse;
  p.rand_attn = rand_attn;
  p.seq_mask = seq_mask;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.H = H;
  p.L = L;
  p.nb = nb;
  p.r = r;
  p.sparse = sparse ? 1 : 0;
  p.out_f32 = out_dtype == BB_OUT_F32 ? 1 : 0;
  p.scale = 1.0f / sqrtf(static_cast<float>(d));
  bigbird_bwd_kernel<<<dim3(nb, B * H), kThreads, smem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? BB_OK : BB_ERR_CUDA;
}
