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
// block receives from every query block that attends to it). Every product
// is computed as 4x4 register tiles per thread (16 x 16 threads over a 64x64
// result), reading 4-wide vectors along the summed dimension, so each shared-
// memory load feeds four FMAs or more.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/bigbird_attn.h"

namespace bbw {

constexpr int kBlock = 64;
constexpr int kDim = 64;
constexpr int kThreads = 256;
constexpr int kLd = kDim + 4;  // row stride of the fp32 tiles (16-byte aligned rows)
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
  const int row = t >> 2;          // row of the D computation (4 threads per row)
  const int c0 = (t & 3) * 16;     // its 16 columns
  const int ty = t >> 4;           // 4x4 result tile: rows (or keys) 4ty..4ty+3
  const int tx = t & 15;           // and columns (keys or dims) 4tx..4tx+3
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

  float dq[4][4];  // rows 4ty.., dims 4tx..
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) dq[a][c] = 0.f;

  for (int e = 0; e < nkb; ++e) {
    const int j = all ? e : s.list[e];
    const size_t k0 = head + static_cast<size_t>(j) * kBlock;
    load_tile(s.k, p.k, k0);
    load_tile(s.v, p.v, k0);
    if (t < kBlock) s.bias[t] = (p.seq_mask && !p.seq_mask[static_cast<size_t>(b) * p.L + j * kBlock + t]) ? -10000.f : 0.f;
    __syncthreads();
    // p and ds for rows 4ty..4ty+3 and keys 4tx..4tx+3 of the block
    {
      float sc[4][4], dp[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) sc[a][c] = dp[a][c] = 0.f;
#pragma unroll 2
      for (int x = 0; x < kDim; x += 4) {
        float4 qa[4], ka[4], da[4], va[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          qa[a] = *reinterpret_cast<const float4*>(&s.q[4 * ty + a][x]);
          da[a] = *reinterpret_cast<const float4*>(&s.dout[4 * ty + a][x]);
          ka[a] = *reinterpret_cast<const float4*>(&s.k[4 * tx + a][x]);
          va[a] = *reinterpret_cast<const float4*>(&s.v[4 * tx + a][x]);
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            sc[a][c] = fmaf(qa[a].x, ka[c].x, fmaf(qa[a].y, ka[c].y, fmaf(qa[a].z, ka[c].z, fmaf(qa[a].w, ka[c].w, sc[a][c]))));
            dp[a][c] = fmaf(da[a].x, va[c].x, fmaf(da[a].y, va[c].y, fmaf(da[a].z, va[c].z, fmaf(da[a].w, va[c].w, dp[a][c]))));
          }
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int rr = 4 * ty + a;
        const float lse2 = s.lse[rr] * log2e;
        const float dr = s.dsum[rr];
        float4 pv4, ds4;
        float* pv = reinterpret_cast<float*>(&pv4);
        float* dsv = reinterpret_cast<float*>(&ds4);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          pv[c] = exp2f(fmaf(sc[a][c], p.scale, s.bias[4 * tx + c]) * log2e - lse2);
          dsv[c] = pv[c] * (dp[a][c] - dr);
        }
        *reinterpret_cast<float4*>(&s.p[rr][4 * tx]) = pv4;
        *reinterpret_cast<float4*>(&s.ds[rr][4 * tx]) = ds4;
      }
    }
    __syncthreads();
    // dq[rows 4ty.., dims 4tx..] += ds[rows, all keys] . k[all keys, dims]
#pragma unroll 4
    for (int c = 0; c < kBlock; ++c) {
      const float4 kv = *reinterpret_cast<const float4*>(&s.k[c][4 * tx]);
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float w = s.ds[4 * ty + a][c];
        dq[a][0] = fmaf(w, kv.x, dq[a][0]);
        dq[a][1] = fmaf(w, kv.y, dq[a][1]);
        dq[a][2] = fmaf(w, kv.z, dq[a][2]);
        dq[a][3] = fmaf(w, kv.w, dq[a][3]);
      }
    }
    // dk[keys 4ty.., dims 4tx..] += ds^T q,  dv[keys 4ty.., dims 4tx..] += p^T dout
    {
      float dk[4][4], dv[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) dk[a][c] = dv[a][c] = 0.f;
#pragma unroll 4
      for (int rr = 0; rr < kBlock; ++rr) {
        const float4 w = *reinterpret_cast<const float4*>(&s.ds[rr][4 * ty]);
        const float4 pw = *reinterpret_cast<const float4*>(&s.p[rr][4 * ty]);
        const float4 qv = *reinterpret_cast<const float4*>(&s.q[rr][4 * tx]);
        const float4 dv4 = *reinterpret_cast<const float4*>(&s.dout[rr][4 * tx]);
        const float ws[4] = {w.x, w.y, w.z, w.w};
        const float ps[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          dk[a][0] = fmaf(ws[a], qv.x, dk[a][0]);
          dk[a][1] = fmaf(ws[a], qv.y, dk[a][1]);
          dk[a][2] = fmaf(ws[a], qv.z, dk[a][2]);
          dk[a][3] = fmaf(ws[a], qv.w, dk[a][3]);
          dv[a][0] = fmaf(ps[a], dv4.x, dv[a][0]);
          dv[a][1] = fmaf(ps[a], dv4.y, dv[a][1]);
          dv[a][2] = fmaf(ps[a], dv4.z, dv[a][2]);
          dv[a][3] = fmaf(ps[a], dv4.w, dv[a][3]);
        }
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        float* dkp = p.dk + (k0 + 4 * ty + a) * kDim + 4 * tx;
        float* dvp = p.dv + (k0 + 4 * ty + a) * kDim + 4 * tx;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          atomicAdd(dkp + c, dk[a][c] * p.scale);
          atomicAdd(dvp + c, dv[a][c]);
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a)
    *reinterpret_cast<float4*>(p.dq + (q0 + 4 * ty + a) * kDim + 4 * tx) =
        make_float4(dq[a][0] * p.scale, dq[a][1] * p.scale, dq[a][2] * p.scale, dq[a][3] * p.scale);
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
