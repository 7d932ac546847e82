/*
 * Sparse brute-force CPU reference of BigBird ITC attention (forward), fp64.
 *
 * TEST AND BENCHMARK INFRASTRUCTURE ONLY (like the rest of oracle/): the
 * product path never links or calls it. It computes only the work the method
 * asks for, so it is the fair CPU timing baseline; tests pin it against the
 * dense-mask NumPy oracle.
 *
 * For every (b, h) and query token t in query block i = t / block:
 *   key blocks of row i [TFG-BigBird, section "BigBird：从二次方注意力到线性稀疏注意力";
 *   HF-Pegasus, section "三类注意力组合"]:
 *     i == 0 or i == nb-1, or the full-attention fallback (nb <= 5 + 2r,
 *     HF-Pegasus, section "序列过短时的自动回退"): every block;
 *     otherwise the set {0, nb-1, i-1, i, i+1} united with rand_attn[h][i-1][0..r)
 *     (a repeated or overlapping entry adds nothing);
 *   s[t, k] = (q_t . k_k) / sqrt(d) + (seq_mask[b, k] ? 0 : -10000) for the keys k
 *   of those blocks; out[t] = sum_k softmax(s)[k] v_k.
 * Inputs are bf16 bit patterns, used at their exact values.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_double(uint16_t x) {
  const uint32_t bits = (uint32_t)x << 16;
  float f;
  memcpy(&f, &bits, sizeof(f));
  return (double)f;
}

/* Returns 0 on success, 1 on bad arguments, 2 on an out-of-range rand_attn entry, 3 on allocation failure. */
int bigbird_sparse_ref(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* rand_attn,
                       const uint8_t* seq_mask, double* out, int B, int H, int L, int d, int block, int r,
                       int force_sparse, int nthreads) {
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0 || block <= 0 || r < 1 || L % block != 0) return 1;
  const int nb = L / block;
  const int sparse = force_sparse || nb > 5 + 2 * r;
  if (sparse && !rand_attn) return 1;
  if (sparse) {
    for (long i = 0; i < (long)H * (nb - 2) * r; ++i)
      if (rand_attn[i] < 0 || rand_attn[i] >= nb) return 2;
  }
  const double scale = 1.0 / sqrt((double)d);
  int status = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
  {
    char* use = (char*)malloc((size_t)nb);
    double* s = (double*)malloc(sizeof(double) * (size_t)L);
    int* keys = (int*)malloc(sizeof(int) * (size_t)L);
    double* qd = (double*)malloc(sizeof(double) * (size_t)d);
    if (!use || !s || !keys || !qd) {
#pragma omp atomic write
      status = 3;
    } else {
#pragma omp for schedule(dynamic, 16)
      for (long task = 0; task < (long)B * H * L; ++task) {
        const int t = (int)(task % L);
        const int h = (int)((task / L) % H);
        const int b = (int)(task / ((long)L * H));
        const int i = t / block;
        const size_t head = ((size_t)b * H + h) * (size_t)L;
        /* the row's key blocks */
        if (!sparse || i == 0 || i == nb - 1) {
          memset(use, 1, (size_t)nb);
        } else {
          memset(use, 0, (size_t)nb);
          use[0] = use[nb - 1] = 1;
          use[i - 1] = use[i] = use[i + 1] = 1;
          for (int e = 0; e < r; ++e) use[rand_attn[((size_t)h * (nb - 2) + (i - 1)) * r + e]] = 1;
        }
        int nk = 0;
        for (int j = 0; j < nb; ++j)
          if (use[j])
            for (int c = 0; c < block; ++c) keys[nk++] = j * block + c;
        /* scores */
        for (int x = 0; x < d; ++x) qd[x] = bf16_to_double(q[(head + t) * d + x]);
        double mx = -INFINITY;
        for (int n = 0; n < nk; ++n) {
          const int kk = keys[n];
          double dot = 0.0;
          for (int x = 0; x < d; ++x) dot += qd[x] * bf16_to_double(k[(head + kk) * d + x]);
          double sv = dot * scale;
          if (seq_mask && !seq_mask[(size_t)b * L + kk]) sv += -10000.0;
          s[n] = sv;
          if (sv > mx) mx = sv;
        }
        /* softmax and weighted sum of V */
        double* o = out + (head + t) * d;
        for (int x = 0; x < d; ++x) o[x] = 0.0;
        double sum = 0.0;
        for (int n = 0; n < nk; ++n) {
          const double p = exp(s[n] - mx);
          sum += p;
          const uint16_t* vr = v + (head + keys[n]) * d;
          for (int x = 0; x < d; ++x) o[x] += p * bf16_to_double(vr[x]);
        }
        for (int x = 0; x < d; ++x) o[x] /= sum;
      }
    }
    free(use);
    free(s);
    free(keys);
    free(qd);
  }
  return status;
}
