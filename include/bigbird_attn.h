/*
 * bigbird_attn.h -- C ABI of the B200 (sm_100a) BigBird ITC block-sparse
 * attention: the forward pass, its host-side preparation routines, the
 * backward pass and the attention-probability export.
 *
 * Pages cited below:
 *   [TFG-BigBird] "models 仓库中的 BigBird：线性复杂度稀疏注意力与长序列训练的完整实践"
 *                 (TensorFlow Model Garden official/projects/bigbird)
 *   [HF-Pegasus]  "BigBirdPegasus 长序列条件生成模型详解从稀疏注意力原理到 Transformers 实战"
 *                 (Hugging Face modeling_bigbird_pegasus.py)
 *
 * Conventions for every entry point:
 *   - Tensors are dense, row-major, with no padding between rows.
 *     Q, K, V, O: [B, H, L, d]; seq_mask: [B, L]; rand_attn: [H, nb-2, r],
 *     where nb = L / block.
 *   - "device" pointers are CUDA global memory of the current device;
 *     "host" pointers are ordinary CPU memory. The caller owns every buffer;
 *     no function keeps a pointer after it returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream). Device work is enqueued asynchronously on it; no entry point
 *     synchronises the stream unless its comment says so.
 *   - Return value: a bb_status. On any error nothing is launched and no
 *     output is written, except BB_ERR_CUDA after a launch.
 */
#ifndef BIGBIRD_ATTN_H
#define BIGBIRD_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BB_OK = 0,
  BB_ERR_INVALID_ARG = 1,   /* NULL pointer, non-positive size, L % block != 0, r < 1 */
  BB_ERR_UNSUPPORTED = 2,   /* unsupported d / block, misaligned pointer, no sm_100 device */
  BB_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
  BB_ERR_BAD_RAND_ATTN = 4, /* rand_attn breaks the generator's rules (validator / debug checks) */
  BB_ERR_DEVICE = 5         /* a kernel reported a device-side error (see bigbird_device_status) */
} bb_status;

/* Output element type of the forward pass. */
enum { BB_OUT_BF16 = 0, BB_OUT_F32 = 1 };

/* Flags of bigbird_attn_fwd_ex. */
enum {
  /* Use the sparse pattern even when nb <= 5 + 2r (requires nb >= 5 + r). */
  BB_FLAG_FORCE_SPARSE = 1u,
  /* Copy rand_attn to the host and validate it before launching; synchronises the stream. */
  BB_FLAG_DEBUG_CHECKS = 2u
};

/*
 * bigbird_attn_fwd -- BigBird ITC block-sparse attention forward, bf16 in, bf16 out.
 *
 * For every (b, h) and query block i (rows i*block .. i*block+block-1):
 *   - i = 0 and i = nb-1 attend to all L keys (global rows)
 *     [TFG-BigBird, section "BigBird：从二次方注意力到线性稀疏注意力"; HF-Pegasus,
 *     section "三类注意力组合"];
 *   - every other i attends to key blocks {0, nb-1} (global), {i-1, i, i+1}
 *     (sliding window) and rand_attn[h][i-1][0..r) (random)
 *     [same sections; TFG-BigBird, section "随机块掩码是如何生成的"].
 * The key set of a row is a set: a random entry equal to a window or global
 * block, or repeated, adds nothing. Scores are (q . k) / sqrt(d), plus -10000
 * for keys with seq_mask == 0 [TFG-BigBird, "BigBird：从二次方注意力到线性稀疏注意力"];
 * out = softmax(scores) . V with fp32 accumulation.
 * If nb <= 5 + 2r the call computes full attention and ignores rand_attn
 * [HF-Pegasus, section "序列过短时的自动回退"].
 *
 *   q, k, v    device, bf16 [B, H, L, d], 16-byte aligned.
 *   rand_attn  device, int32 [H, nb-2, r]; entries must lie in [0, nb) (an
 *              entry outside is skipped and flagged in bigbird_device_status).
 *              May be NULL only in the full-attention fallback.
 *   seq_mask   device, uint8 [B, L], nonzero = valid key; NULL = all valid.
 *   out        device, bf16 [B, H, L, d], 16-byte aligned; must not alias q/k/v.
 *   B, H, L, d, block, r  sizes: d in {64, 128}, block in {32, 64, 128}.
 *              Blocks of 64 or 128 at d 64 or 128 run the tensor-core kernel
 *              (64-token tiles: a block of 128 is two; d 128 is two 64-column
 *              chunks per row); block 32, and full attention over more than
 *              42 tiles (block 128 with r > 8), run a CUDA-core kernel (fp32
 *              arithmetic, one CTA per query block, no workspace) with the
 *              same results.
 *   stream     cudaStream_t.
 * Errors: BB_ERR_INVALID_ARG for L % block != 0 [HF-Pegasus, section
 * "序列长度的块对齐要求"] or r < 1 [HF-Pegasus, section "使用限制与注意事项"];
 * BB_ERR_UNSUPPORTED for other d/block or misalignment. Every finite bf16
 * value is taken. On the tensor-core kernel P.V runs in fp16 (P and V converted in
 * shared memory); when V holds a value of magnitude >= 65536, which fp16
 * cannot represent, the call is done again with bf16 P and V (8 significant
 * bits of P instead of 11), which about doubles its time. A call launches the
 * fp16 kernel, then its bf16 instance as its programmatic dependent: that
 * grid merges the key ranges of the split global rows (when the recompute is
 * needed, after doing the call again) and otherwise returns at once.
 * The workspace (the work-unit counters and,
 * for split global rows, their partial results; see
 * bigbird_attn_workspace_size) is taken with cudaMallocAsync on `stream`,
 * zeroed with cudaMemsetAsync and released with cudaFreeAsync: callers that
 * must not allocate use bigbird_attn_fwd_ex with their own workspace, or
 * bigbird_attn_fwd_noalloc.
 */
int bigbird_attn_fwd(const void* q, const void* k, const void* v, const int32_t* rand_attn,
                     const uint8_t* seq_mask, void* out, int B, int H, int L, int d, int block, int r,
                     void* stream);

/*
 * Bytes of device workspace bigbird_attn_fwd_ex needs for these sizes and
 * flags (0 if the sizes are invalid, and for the sizes the CUDA-core kernel
 * runs, which need none). For the tensor-core kernel it starts with 256 bytes of
 * counters: the one through which the CTAs share out the work units, one that
 * finds the CTA finishing last (which sets the counters back to zero), and
 * the flag that asks for the bf16 recompute (cleared by the bf16 instance when
 * it runs). When the global rows are split into key ranges (sparse pattern:
 * ranges of 8 tiles of 64 keys; 12 tiles at block 64, d 64 when the sequence
 * has 256 or more tiles) each range's partial result follows, per
 * global unit (one unit holds both global blocks at block 64, one unit per
 * global block at block 128): output normalised by its own sum [128 rows, d],
 * running max and running sum, merged by log-sum-exp by the bf16 instance.
 * A fourth counter (the ranges the bf16 instance has redone) is used only on
 * the recompute path and is zero between calls like the others.
 */
size_t bigbird_attn_workspace_size(int B, int H, int L, int d, int block, int r, unsigned flags);

/*
 * bigbird_attn_fwd_ex -- bigbird_attn_fwd with an output type, flags and an
 * optional caller-provided workspace.
 *   out_dtype  BB_OUT_BF16 (out is bf16) or BB_OUT_F32 (out is fp32 [B,H,L,d]).
 *   flags      BB_FLAG_* bits.
 *   workspace  device, 256-byte aligned, at least
 *              bigbird_attn_workspace_size(...) bytes, zero-filled before
 *              its first use; every call that completes leaves its counters
 *              at zero again, so a workspace is reused without clearing it.
 *              NULL = allocate and zero one with cudaMallocAsync /
 *              cudaMemsetAsync on `stream` (freed with cudaFreeAsync after
 *              the launch). Calls that share a workspace must not overlap on
 *              the GPU.
 */
int bigbird_attn_fwd_ex(const void* q, const void* k, const void* v, const int32_t* rand_attn,
                        const uint8_t* seq_mask, void* out, int B, int H, int L, int d, int block, int r,
                        int out_dtype, unsigned flags, void* workspace, size_t workspace_bytes, void* stream);

/*
 * bigbird_attn_fwd_host -- bigbird_attn_fwd_ex with q, k, v, rand_attn,
 * seq_mask and out in HOST memory (page-locked for the copies to overlap):
 * layouts as bigbird_attn_fwd_ex, out bf16 or fp32 per out_dtype. The batch
 * goes through the GPU one sequence at a time in two device slots, on three
 * streams of the library's own (copies in, the forward, copies out), so that
 * copying sequence b+1 in, computing b and copying b-1 out overlap; the
 * results are those of bigbird_attn_fwd_ex on the whole batch, bit for bit.
 *   scratch  device, 256-byte aligned, at least
 *            bigbird_attn_fwd_host_scratch_bytes(...) bytes; no initialisation
 *            needed (the call zeroes the workspace counters it uses).
 *   stream   the caller's stream: the call starts after the work queued on it
 *            and the stream waits for the call's last copy; synchronise it
 *            before reading out.
 * Calls for one device are enqueued one at a time (a mutex); calls that share
 * a scratch must not overlap on the GPU. Errors as bigbird_attn_fwd_ex
 * (BB_FLAG_DEBUG_CHECKS is ignored: rand_attn is on the host already).
 */
int bigbird_attn_fwd_host(const void* q, const void* k, const void* v, const int32_t* rand_attn,
                          const uint8_t* seq_mask, void* out, int B, int H, int L, int d, int block, int r,
                          int out_dtype, unsigned flags, void* scratch, size_t scratch_bytes, void* stream);

/* Bytes of device scratch bigbird_attn_fwd_host needs (0 if the sizes are invalid). */
size_t bigbird_attn_fwd_host_scratch_bytes(int B, int H, int L, int d, int block, int r, unsigned flags);

/*
 * bigbird_attn_fwd_train -- bigbird_attn_fwd_ex that also writes, for the
 * backward pass, each row's natural-log log-sum-exp of its scores:
 *   lse[b,h,t] = log sum_k exp(s[t,k]),  s = q.k / sqrt(d) + bias
 * over the row's attended keys (the softmax normaliser).
 *   lse  device fp32 [B, H, L], written in full; NULL -> BB_ERR_INVALID_ARG.
 * Everything else as bigbird_attn_fwd_ex.
 */
int bigbird_attn_fwd_train(const void* q, const void* k, const void* v, const int32_t* rand_attn,
                           const uint8_t* seq_mask, void* out, float* lse, int B, int H, int L, int d, int block,
                           int r, int out_dtype, unsigned flags, void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * bigbird_attn_bwd -- gradients of sum(dout * out) with respect to q, k, v
 * for the same pattern as the forward [TFG-BigBird, section "BigBird：从二次方
 * 注意力到线性稀疏注意力"; HF-Pegasus, section "三类注意力组合"], by the chain rule
 * through each row's softmax (p recomputed as exp(s - lse)):
 *   dv = p^T dout,  dp = dout v^T,  ds = p (dp - rowsum(dout * out)),
 *   dq = ds k / sqrt(d),  dk = ds^T q / sqrt(d).
 *   q, k, v, dout  device bf16 [B, H, L, d] (dout: gradient of out), 16-byte aligned.
 *   out            device [B, H, L, d]: the forward's output, bf16 or fp32 (out_dtype).
 *   lse            device fp32 [B, H, L] from bigbird_attn_fwd_train.
 *   rand_attn, seq_mask, B, H, L, d, block, r, BB_FLAG_FORCE_SPARSE: as the forward.
 *   dq, dk, dv     device fp32 [B, H, L, d], written in full, 16-byte aligned.
 * Tensor cores (tcgen05, bf16 operands, fp32 accumulation): a row-dot
 * kernel (D = rowsum(dout * out)), a query-stationary dq kernel, a
 * key-stationary dk/dv kernel and, when the global rows are split into key
 * ranges, a kernel summing their partial results -- no atomics, so the
 * gradients are the same bit for bit on every run. The workspace (counters,
 * D and the partial sums; bigbird_attn_bwd_workspace_size) is taken with
 * cudaMallocAsync on `stream`, its counters zeroed with cudaMemsetAsync, and
 * released with cudaFreeAsync; bigbird_attn_bwd_ex takes the caller's.
 * Sizes: d 64 or 128, block 64 or 128 (a block of 128 is two 64-token tiles,
 * d 128 two 64-column chunks; at d 128 one CTA per SM); other sizes, and full
 * attention over more than 42 tiles (block 128 with r > 8), return
 * BB_ERR_UNSUPPORTED. Asynchronous on `stream`. Other errors as the forward.
 * Out-of-range rand_attn entries are skipped and flagged in
 * bigbird_device_status.
 */
int bigbird_attn_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
                     const float* lse, const int32_t* rand_attn, const uint8_t* seq_mask, float* dq, float* dk,
                     float* dv, int B, int H, int L, int d, int block, int r, int out_dtype, unsigned flags,
                     void* stream);

/*
 * Bytes of device workspace bigbird_attn_bwd_ex needs (0 for invalid or
 * unsupported sizes): 256 bytes of counters, D [B*H*L] fp32 (rounded up to
 * 256 bytes) and, when the global rows are split into key ranges (sparse
 * pattern), three partial-sum arrays [B*H, n_glob * ceil(L / 512), 128, d]
 * fp32 (dq of the global query blocks, dv and dk of the global key blocks;
 * n_glob = 1 at block 64, where one unit holds both global blocks, 2 at
 * block 128).
 */
size_t bigbird_attn_bwd_workspace_size(int B, int H, int L, int d, int block, int r, unsigned flags);

/*
 * bigbird_attn_bwd_ex -- bigbird_attn_bwd with a caller-provided workspace:
 * device, 256-byte aligned, at least bigbird_attn_bwd_workspace_size(...)
 * bytes, zero-filled before its first use (every call that completes leaves
 * its counters at zero again); NULL allocates one as bigbird_attn_bwd does.
 * Calls that share a workspace must not overlap on the GPU.
 */
int bigbird_attn_bwd_ex(const void* q, const void* k, const void* v, const void* out, const void* dout,
                        const float* lse, const int32_t* rand_attn, const uint8_t* seq_mask, float* dq, float* dk,
                        float* dv, int B, int H, int L, int d, int block, int r, int out_dtype, unsigned flags,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * Attention probabilities (the output_attentions path). The block-sparse model
 * writes each row group's softmax weights into a full [B, H, L, L] matrix that
 * is zero outside the pattern [HF-Pegasus, section "三类注意力组合": four
 * scatter_ calls]; the matrix carries no gradient [HF-Pegasus, section
 * "使用限制与注意事项"]. These calls recompute the weights from q, k and the
 * row log-sum-exp that bigbird_attn_fwd_train wrote for the same inputs:
 *   p[b,h,t,k] = exp(q_t.k_k / sqrt(d) + bias_k - lse[b,h,t])
 * on the row's attended keys (bias_k = -10000 for a padded key), 0 elsewhere.
 *
 * bigbird_attn_probs_layout -- shapes of the packed layout (host, no GPU):
 *   *global_rows  G: 2 in the sparse mode (query blocks 0 and nb-1), nb in the
 *                 full-attention fallback;
 *   *band_rows    nb - 2 in the sparse mode, 0 in the fallback;
 *   *band_slots   5 + r in the sparse mode, 0 in the fallback.
 * Any output pointer may be NULL. Errors as bigbird_attn_fwd_ex's arguments.
 *
 * bigbird_attn_probs -- the weights in the packed block-sparse layout:
 *   q, k          device bf16 [B, H, L, d]; lse device fp32 [B, H, L];
 *   rand_attn, seq_mask, B, H, L, d, block, r, BB_FLAG_FORCE_SPARSE: as the forward;
 *   probs_global  device [B, H, G, 64, L]: row g's weights over every key
 *                 (g = 0: query block 0, g = 1: query block nb-1; in the
 *                 fallback g = every query block, i.e. the whole matrix);
 *   probs_band    device [B, H, nb-2, 5+r, 64, 64]: tile t of query block i
 *                 (1 <= i <= nb-2) holds its weights against key block
 *                 bigbird_pattern_table(...)[h][i-1][t]; tiles whose table
 *                 entry is -1 are written as zeros. Unused (may be NULL) in
 *                 the fallback;
 *   out_dtype     BB_OUT_F32 or BB_OUT_BF16 (both outputs).
 * Every element of both outputs is written. Asynchronous on `stream`; nothing
 * is allocated. Output pointers must be 16-byte aligned
 * (BB_ERR_UNSUPPORTED otherwise). Out-of-range rand_attn entries are skipped
 * and flagged (bit 1 of bigbird_device_status). Rows whose keys are all
 * padded are accurate to ~1e-3 relative (their lse sits near -10000, where
 * fp32 keeps ~3 decimal places); every other row to ~1e-5.
 *
 * bigbird_attn_probs_dense -- the same weights scattered into the full
 * matrix: probs device [B, H, L, L] (B*H*L*L elements of out_dtype), zeros
 * outside the pattern, every element written.
 */
int bigbird_attn_probs_layout(int L, int d, int block, int r, unsigned flags, int* global_rows, int* band_rows,
                              int* band_slots);
int bigbird_attn_probs(const void* q, const void* k, const float* lse, const int32_t* rand_attn,
                       const uint8_t* seq_mask, void* probs_global, void* probs_band, int B, int H, int L, int d,
                       int block, int r, int out_dtype, unsigned flags, void* stream);
int bigbird_attn_probs_dense(const void* q, const void* k, const float* lse, const int32_t* rand_attn,
                             const uint8_t* seq_mask, void* probs, int B, int H, int L, int d, int block, int r,
                             int out_dtype, unsigned flags, void* stream);

/*
 * bigbird_wait_probe -- self-test of the failure-detection path. Launches one
 * thread that waits, with the same bounded wait the kernels use, for an
 * mbarrier nothing arrives on; after limit_us microseconds (1 .. 2e6) the
 * wait gives up and sets the timeout bit (2) of the device status word, as
 * a lost completion inside bigbird_attn_fwd would. Nothing faults or hangs;
 * read the bit with bigbird_device_status. Returns BB_OK once launched,
 * BB_ERR_INVALID_ARG for a limit out of range.
 */
int bigbird_wait_probe(unsigned limit_us, void* stream);

/* 1 if (L, block, r) runs full attention (nb <= 5 + 2r), 0 if sparse, <0 on
 * invalid sizes [HF-Pegasus, section "序列过短时的自动回退"]. */
int bigbird_attn_is_fallback(int L, int block, int r);

/*
 * bigbird_rand_attn_generate -- seeded random adjacency (host).
 *   host_out  host, int32 [H, nb-2, r]; row i-1 holds query block i's random blocks.
 * Row i draws a uniformly random r-subset, in random order, of its candidate
 * pool: blocks 1..nb-2 without i-1, i, i+1 [TFG-BigBird, section
 * "随机块掩码是如何生成的"]; with last_idx > 0 only blocks j with
 * (j+1)*block <= last_idx qualify (the page's last_idx = 1024 cap; 0 = off).
 * The draw is a partial Fisher-Yates shuffle of the ascending pool; draw t of
 * row (h, i) takes the SplitMix64 output of state `seed` at counter
 * ((h*(nb-2) + i-1) << 20) + 1 + t' (t' counts the row's draws, rejections
 * included), bounded without bias by rejecting u < (2^64 - n) mod n.
 * Deterministic for a given seed; heads get distinct streams.
 * Errors: BB_ERR_INVALID_ARG for bad sizes or a row with fewer than r candidates.
 */
int bigbird_rand_attn_generate(int32_t* host_out, int H, int L, int block, int r, uint64_t seed, int last_idx);

/*
 * bigbird_rand_attn_validate -- check a host rand_attn [H, nb-2, r] against the
 * generator's rules: every entry a candidate of its row (range, not in the
 * row's window or global blocks, before last_idx when > 0) and no repeats
 * within a row [TFG-BigBird, section "随机块掩码是如何生成的"].
 * Returns BB_OK or BB_ERR_BAD_RAND_ATTN (BB_ERR_INVALID_ARG for bad sizes).
 */
int bigbird_rand_attn_validate(const int32_t* host_ra, int H, int L, int block, int r, int last_idx);

/*
 * bigbird_mask_prep -- the BigBirdMasks tensors from a [B, L] mask (host)
 * [TFG-BigBird, section "随机块掩码是如何生成的", the four-mask tuple]:
 *   blocked   host uint8 [B, nb, block]          seq_mask cut into blocks
 *   band      host uint8 [B, nb-4, block, 3*block]
 *             band[b, i-2, x, w*block + y] = m[b, i*block + x] * m[b, (i-1+w)*block + y]
 *             for middle query block i in [2, nb-3], window slot w in {0,1,2}
 *   from_mask host uint8 [B, L] (query side), to_mask host uint8 [B, L] (key side)
 * Output values are 0/1. Any output pointer may be NULL to skip it. Requires nb >= 4.
 */
int bigbird_mask_prep(const uint8_t* seq_mask, int B, int L, int block, uint8_t* blocked, uint8_t* band,
                      uint8_t* from_mask, uint8_t* to_mask);

/*
 * bigbird_pattern_table -- the sparse pattern as lists (host):
 *   out  host int32 [H, nb-2, 5+r]; row i-1 lists query block i's distinct key
 *        blocks in ascending order, padded with -1. Rows 0 and nb-1 attend to
 *        every block and are not listed.
 * Entries of host_ra outside [0, nb) give BB_ERR_BAD_RAND_ATTN.
 */
int bigbird_pattern_table(const int32_t* host_ra, int H, int L, int block, int r, int32_t* out);

/*
 * bigbird_device_status -- read and clear the library's device error word
 * after synchronising `stream`. Bit 1: a rand_attn entry outside [0, nb) was
 * skipped; bit 2: a kernel wait timed out (a lost completion). *host_status
 * receives the word. Returns BB_OK, or BB_ERR_CUDA if the copy failed.
 * The word is one per device and process: every call of every entry point,
 * on any stream and from any host thread, ORs its bits into the same word,
 * and a read clears the bits of all of them. Read it where no other work of
 * this library is in flight on the device, or attribute its bits to all the
 * calls since the previous read.
 */
int bigbird_device_status(void* stream, uint32_t* host_status);

/*
 * bigbird_attn_fwd_noalloc -- bigbird_attn_fwd_ex without any device memory
 * allocation. (The pages have no counterpart: this entry point exists for
 * callers that cannot allocate device memory while they run, e.g. a server or
 * real-time loop that reserves all GPU memory at start-up and must not hit the
 * allocator, or its device-wide synchronisation, inside a step.)
 *
 * The workspace (counters and the split global rows' partial results) comes
 * from a fixed region of bigbird_attn_noalloc_scratch_bytes() bytes (32 MiB)
 * that the library's module holds on every GPU that loads it, until the
 * process exits. Arguments and
 * results are those of bigbird_attn_fwd_ex, except:
 *   - there is no workspace argument;
 *   - a problem whose scratch need (bigbird_attn_workspace_size) exceeds the
 *     fixed region returns BB_ERR_UNSUPPORTED before anything is launched
 *     (32 MiB covers, e.g., B*H = 48 heads at L = 4096 or 8 heads at L = 32768);
 *   - BB_FLAG_DEBUG_CHECKS returns BB_ERR_UNSUPPORTED (that check allocates a
 *     host buffer).
 * The first call on a device looks up the region's device address (once per
 * device, with that device current); make that first call before any stream
 * capture. All calls share the one region, which keeps what the previous
 * call left: each call first clears the counters at its start with
 * cudaMemsetAsync on `stream` (the partial results are rewritten before they
 * are read). Calls that overlap on the GPU -- on different streams, or from
 * different threads -- race on the region.
 */
int bigbird_attn_fwd_noalloc(const void* q, const void* k, const void* v, const int32_t* rand_attn,
                             const uint8_t* seq_mask, void* out, int B, int H, int L, int d, int block, int r,
                             int out_dtype, unsigned flags, void* stream);

/* Size in bytes of the fixed scratch region of bigbird_attn_fwd_noalloc. */
size_t bigbird_attn_noalloc_scratch_bytes(void);

/* Static, human-readable text of a bb_status. */
const char* bigbird_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* BIGBIRD_ATTN_H */
