// Host-side preparation of the BigBird ITC pattern: the seeded random-block
// generator and its validator, the BigBirdMasks tensors and the pattern table.
// Declarations and argument contracts: include/bigbird_attn.h.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <vector>

#include "../../include/bigbird_attn.h"

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;
constexpr int kRowCounterShift = 20;

// SplitMix64 output function (Steele, Lea & Flood, OOPSLA 2014).
inline uint64_t splitmix64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// n-th output (n >= 1) of the SplitMix64 stream whose state starts at seed.
inline uint64_t splitmix64_at(uint64_t seed, uint64_t n) { return splitmix64_mix(seed + n * kGamma); }

bool sizes_ok(int L, int block, int r) { return L > 0 && block > 0 && r >= 1 && L % block == 0; }

// Candidate random blocks of query block row i [TFG-BigBird, "随机块掩码是如何生成的"]:
// the middle blocks 1..nb-2 without the row's window i-1, i, i+1, and, when
// last_idx > 0, only blocks lying wholly before token last_idx.
void candidate_pool(int i, int nb, int block, int last_idx, std::vector<int32_t>& pool) {
  pool.clear();
  for (int j = 1; j <= nb - 2; ++j) {
    if (j >= i - 1 && j <= i + 1) continue;
    if (last_idx > 0 && static_cast<int64_t>(j + 1) * block > last_idx) continue;
    pool.push_back(j);
  }
}

}  // namespace

extern "C" {

int bigbird_attn_is_fallback(int L, int block, int r) {
  if (!sizes_ok(L, block, r)) return -1;
  return (L / block) <= 5 + 2 * r ? 1 : 0;
}

int bigbird_rand_attn_generate(int32_t* host_out, int H, int L, int block, int r, uint64_t seed, int last_idx) {
  if (!host_out || H <= 0 || !sizes_ok(L, block, r) || last_idx < 0) return BB_ERR_INVALID_ARG;
  const int nb = L / block;
  if (nb < 3) return BB_ERR_INVALID_ARG;
  std::vector<int32_t> pool;
  // Check feasibility of every row first so that nothing is written on error.
  for (int i = 1; i <= nb - 2; ++i) {
    candidate_pool(i, nb, block, last_idx, pool);
    if (static_cast<int>(pool.size()) < r) return BB_ERR_INVALID_ARG;
  }
  for (int h = 0; h < H; ++h) {
    for (int i = 1; i <= nb - 2; ++i) {
      candidate_pool(i, nb, block, last_idx, pool);
      const uint64_t n = pool.size();
      uint64_t ctr = (static_cast<uint64_t>(h) * static_cast<uint64_t>(nb - 2) + static_cast<uint64_t>(i - 1))
                     << kRowCounterShift;
      int32_t* row = host_out + (static_cast<size_t>(h) * (nb - 2) + (i - 1)) * r;
      for (int t = 0; t < r; ++t) {
        const uint64_t bound = n - static_cast<uint64_t>(t);
        const uint64_t thresh = (0 - bound) % bound;  // 2^64 mod bound
        uint64_t u;
        do {
          u = splitmix64_at(seed, ++ctr);
        } while (u < thresh);
        const uint64_t j = static_cast<uint64_t>(t) + u % bound;
        std::swap(pool[t], pool[j]);
        row[t] = pool[t];
      }
    }
  }
  return BB_OK;
}

int bigbird_rand_attn_validate(const int32_t* host_ra, int H, int L, int block, int r, int last_idx) {
  if (!host_ra || H <= 0 || !sizes_ok(L, block, r) || last_idx < 0) return BB_ERR_INVALID_ARG;
  const int nb = L / block;
  if (nb < 3) return BB_ERR_INVALID_ARG;
  for (int h = 0; h < H; ++h) {
    for (int i = 1; i <= nb - 2; ++i) {
      const int32_t* row = host_ra + (static_cast<size_t>(h) * (nb - 2) + (i - 1)) * r;
      for (int t = 0; t < r; ++t) {
        const int32_t x = row[t];
        if (x < 1 || x > nb - 2) return BB_ERR_BAD_RAND_ATTN;
        if (x >= i - 1 && x <= i + 1) return BB_ERR_BAD_RAND_ATTN;
        if (last_idx > 0 && static_cast<int64_t>(x + 1) * block > last_idx) return BB_ERR_BAD_RAND_ATTN;
        for (int u = 0; u < t; ++u)
          if (row[u] == x) return BB_ERR_BAD_RAND_ATTN;
      }
    }
  }
  return BB_OK;
}

int bigbird_mask_prep(const uint8_t* seq_mask, int B, int L, int block, uint8_t* blocked, uint8_t* band,
                      uint8_t* from_mask, uint8_t* to_mask) {
  if (!seq_mask || B <= 0 || L <= 0 || block <= 0 || L % block != 0) return BB_ERR_INVALID_ARG;
  const int nb = L / block;
  if (nb < 4) return BB_ERR_INVALID_ARG;
  const size_t BL = static_cast<size_t>(B) * L;
  // blocked [B, nb, block] has the same element order as [B, L].
  for (size_t t = 0; t < BL; ++t) {
    const uint8_t m = seq_mask[t] != 0;
    if (blocked) blocked[t] = m;
    if (from_mask) from_mask[t] = m;
    if (to_mask) to_mask[t] = m;
  }
  if (band) {
    const int nmid = nb - 4;
    const size_t row_w = 3 * static_cast<size_t>(block);
    for (int b = 0; b < B; ++b) {
      const uint8_t* m = seq_mask + static_cast<size_t>(b) * L;
      for (int i = 2; i <= nb - 3; ++i) {
        uint8_t* dst = band + ((static_cast<size_t>(b) * nmid + (i - 2)) * block) * row_w;
        for (int x = 0; x < block; ++x) {
          const uint8_t fq = m[static_cast<size_t>(i) * block + x] != 0;
          for (int w = 0; w < 3; ++w) {
            const uint8_t* kb = m + static_cast<size_t>(i - 1 + w) * block;
            uint8_t* o = dst + x * row_w + static_cast<size_t>(w) * block;
            for (int y = 0; y < block; ++y) o[y] = fq & static_cast<uint8_t>(kb[y] != 0);
          }
        }
      }
    }
  }
  return BB_OK;
}

int bigbird_pattern_table(const int32_t* host_ra, int H, int L, int block, int r, int32_t* out) {
  if (!host_ra || !out || H <= 0 || !sizes_ok(L, block, r)) return BB_ERR_INVALID_ARG;
  const int nb = L / block;
  if (nb < 3) return BB_ERR_INVALID_ARG;
  const size_t nrow = static_cast<size_t>(H) * (nb - 2);
  for (size_t t = 0; t < nrow * r; ++t)
    if (host_ra[t] < 0 || host_ra[t] >= nb) return BB_ERR_BAD_RAND_ATTN;
  std::vector<int32_t> s;
  for (int h = 0; h < H; ++h) {
    for (int i = 1; i <= nb - 2; ++i) {
      const int32_t* ra = host_ra + (static_cast<size_t>(h) * (nb - 2) + (i - 1)) * r;
      s.assign({0, nb - 1, i - 1, i, i + 1});
      s.insert(s.end(), ra, ra + r);
      std::sort(s.begin(), s.end());
      s.erase(std::unique(s.begin(), s.end()), s.end());
      int32_t* o = out + (static_cast<size_t>(h) * (nb - 2) + (i - 1)) * (5 + r);
      for (int t = 0; t < 5 + r; ++t) o[t] = t < static_cast<int>(s.size()) ? s[t] : -1;
    }
  }
  return BB_OK;
}

const char* bigbird_status_string(int status) {
  switch (status) {
    case BB_OK: return "ok";
    case BB_ERR_INVALID_ARG: return "invalid argument";
    case BB_ERR_UNSUPPORTED: return "unsupported configuration";
    case BB_ERR_CUDA: return "CUDA error";
    case BB_ERR_BAD_RAND_ATTN: return "rand_attn breaks the random-block rules";
    case BB_ERR_DEVICE: return "device-side error reported by a kernel";
    default: return "unknown status";
  }
}

}  // extern "C"
