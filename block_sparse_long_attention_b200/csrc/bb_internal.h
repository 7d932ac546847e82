// Host-side helpers shared by the library's translation units (not part of
// the C ABI). Implemented in bigbird_attn.cu.
#pragma once

#include <cuda.h>

#include <cstdint>

namespace bb {

// Tensor map over a [rows, 64] bf16 matrix with 64x64 boxes and 128-byte
// swizzle (one box = one block of one head). False if the driver entry point
// is missing or the encoding is rejected.
bool make_tile_map(CUtensorMap* map, const void* base, uint64_t rows);
// The same over a [rows, d] matrix (d = 64 or 128): 64x64 boxes, one per
// 64-column chunk (x = 64 c).
bool make_tile_map_d(CUtensorMap* map, const void* base, uint64_t rows, int d);
// Tensor map over a [rows, 64] fp32 matrix with boxes of 64 rows x 32 columns
// (128 bytes) and 128-byte swizzle, for TMA stores of gradient tiles.
bool make_f32_map(CUtensorMap* map, const void* base, uint64_t rows);

// Device address of the library's status word on the current device `dev`
// (bit 1: an out-of-range rand_attn entry was skipped; bit 2: a bounded wait
// timed out), or null if `dev` is not an sm_100 device or a query failed.
uint32_t* status_word(int dev);

// The CUDA-core forward for the sizes the tensor-core kernel does not take
// (bigbird_generic.cu): supported when d is 64 or 128 and block is 32, 64 or
// 128, except d = block = 64. Arguments and results as bigbird_attn_fwd_train
// with lse optional (null: not written); no workspace.
bool generic_fwd_supported(int d, int block);
int generic_fwd(const void* q, const void* k, const void* v, const int32_t* rand_attn, const uint8_t* seq_mask,
                void* out, float* lse, int B, int H, int L, int d, int block, int r, int out_dtype, unsigned flags,
                void* stream);

}  // namespace bb
