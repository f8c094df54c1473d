/*
 * patch.h - C ABI of libpatch.so, the B200 (sm_100a) implementation of the
 * inference hot path of PATCH, the hybrid tile-sparse linear layer
 *
 *     Y[m][n] = sum_k X[m][k] * W_eff[n][k]        (Y = X * W_eff^T)
 *
 * Source: "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs"
 * (arXiv 2509.23410), as summarised on gist.science/paper/2509.23410:
 *   - section 2 "Methodology: PATCH", "Core Mechanism": W is cut into tiles,
 *     each tile is dense (0% sparsity) or 2:4 sparse (50% sparsity); the
 *     final mask is a combination of a dense and a 2:4 option;
 *   - "Learnable Distributions": a 2-way tile logit distribution chooses
 *     dense vs sparse; inside sparse tiles a separate distribution chooses one
 *     of the 6 possible 2:4 patterns;
 *   - "Inference & Deployment": 128 x 128 execution tiles; dense tiles run on
 *     dense tensor-core MMA, sparse tiles on the 2:4 sparse tensor cores.
 *
 * Conventions shared by every entry point
 *   - bf16 values travel as uint16_t bit patterns.
 *   - W is N x K row-major (K contiguous), X is M x K row-major, Y is M x N
 *     row-major.  N and K must be positive multiples of 128.
 *   - Tiles are numbered row-major: t = tn*Tk + tk, Tn = N/128, Tk = K/128.
 *   - Groups of 4 run along K: group g of row n covers k = 4g .. 4g+3.
 *   - Pattern ids number the kept pair (i0, i1), i0 < i1, lexicographically:
 *       0:(0,1) 1:(0,2) 2:(0,3) 3:(1,2) 4:(1,3) 5:(2,3).
 *   - Every pointer argument except the patch_weight struct itself and the
 *     size outputs of *_sizes / *_workspace_size is a DEVICE pointer.  The
 *     caller allocates and owns every buffer; the library allocates no device
 *     memory, keeps no state between calls and never synchronises the stream
 *     (except patch_read_status).  All calls are asynchronous on `stream`
 *     (a cudaStream_t; NULL = the legacy default stream).
 *   - Host-detectable errors (shape, alignment, null pointer, workspace too
 *     small, not an sm_100 device) return immediately without launching.
 *   - Errors found on the device are OR-ed into the int32 word *dev_status
 *     (PATCH_DEV_* bits); read it with patch_read_status.  dev_status must be
 *     a valid device pointer; the library never clears it.
 *
 * Packed weight format (this library's specification; the paper fixes none)
 *   - Descriptor table: one patch_tile_desc (16 bytes) per tile, row-major.
 *   - Values blob: a sequence of panels; a panel is 128 rows x 64 bf16, row
 *     major with 128-byte rows (16384 bytes).  A dense tile occupies 2 panels
 *     (the tile's k 0..63, then k 64..127).  A sparse tile occupies 1 panel in
 *     which row r holds, for each group g = 0..31, its two kept values in
 *     ascending k at positions 2g and 2g+1.
 *   - Metadata blob: 2048 bytes per sparse tile, at sparse_ordinal*2048.
 *     Group g of tile row r has the 4-bit code i0 | (i1 << 2), stored in the
 *     low nibble of its byte when g is even and the high nibble when g is
 *     odd; the byte is
 *         ((g>>1)&1) | ((r>>3)&1)<<1 | (g>>3)<<2 | (r&7)<<4
 *         | ((g>>2)&1)<<7 | (r>>4)<<8.
 *     This is the order in which the 16-bit sparse tensor-core MMA (M = 128)
 *     reads its metadata from tensor memory after a 128x128b copy (16 bytes
 *     per tensor-memory lane, 4 bytes per 32-K column), so the GEMM moves it
 *     without reshuffling.
 *   - All blobs must be 16-byte aligned.
 */
#ifndef PATCH_H
#define PATCH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define PATCH_API __attribute__((visibility("default")))
#else
#define PATCH_API
#endif

#define PATCH_TILE 128
#define PATCH_PANEL_BYTES 16384
#define PATCH_DENSE_TILE_BYTES 32768
#define PATCH_SPARSE_TILE_BYTES 16384
#define PATCH_META_TILE_BYTES 2048
#define PATCH_DECODE_MAX_M 16

typedef enum {
    PATCH_OK = 0,
    PATCH_ERR_INVALID_ARG = 1, /* null pointer, M < 0, bad path selector */
    PATCH_ERR_SHAPE = 2,       /* N or K not a positive multiple of 128 */
    PATCH_ERR_ALIGN = 3,       /* a pointer not 16-byte aligned */
    PATCH_ERR_DEVICE = 4,      /* current device is not compute capability 10.x */
    PATCH_ERR_CUDA = 5,        /* a CUDA runtime or driver call failed */
    PATCH_ERR_BAD_PATTERN = 6, /* device: pattern id > 5 inside a sparse tile */
    PATCH_ERR_TIMEOUT = 7,     /* device: a bounded wait in a kernel ran out */
    PATCH_ERR_WORKSPACE = 8,   /* workspace pointer null or too small */
    PATCH_ERR_COUNT = 9,       /* device: bitmap's sparse-tile count != n_sparse */
    PATCH_ERR_BOUNDS = 10      /* device: a packed weight breaks the format (patch_check_weight) */
} patch_status_t;

/* Bits OR-ed into *dev_status by the kernels. */
#define PATCH_DEV_BAD_PATTERN 0x1
#define PATCH_DEV_TIMEOUT 0x2
#define PATCH_DEV_COUNT 0x4
#define PATCH_DEV_BOUNDS 0x8

/* Path selector of patch_gemm_ex. */
#define PATCH_PATH_AUTO 0    /* M <= PATCH_DECODE_MAX_M: decode (CUDA-core when N > 524288), else prefill */
#define PATCH_PATH_DECODE 1  /* stream-K weight streaming kernel (TMA + tcgen05, N = 16), M in 1..16, N <= 524288 */
#define PATCH_PATH_PREFILL 2 /* TMA + tcgen05 (dense and 2:4 sparse MMA), any M >= 1 */
#define PATCH_PATH_DECODE_SIMT 3 /* split-K GEMV on CUDA cores (16-byte loads, fp32 FMA), M in 1..16 */
/* Test hook, OR-ed into PATCH_PATH_PREFILL: the prefill producer stops after
 * its first K-tile, so the consumers' bounded waits run out and the kernel
 * reports PATCH_DEV_TIMEOUT and exits cleanly (needs K >= 256 or several
 * output tiles).  Used only to test the timeout path. */
#define PATCH_PATH_TEST_STALL 0x100

/* One descriptor per 128 x 128 tile (16 bytes). */
typedef struct {
    uint32_t kind;           /* 0 = dense, 1 = 2:4 sparse */
    uint32_t sparse_ordinal; /* index of this tile among sparse tiles; 0xFFFFFFFF if dense */
    uint64_t val_offset;     /* byte offset of the tile's first panel in the values blob */
} patch_tile_desc;

/* A packed weight: host struct of device pointers, all owned by the caller. */
typedef struct {
    int64_t N, K;                /* logical shape of W */
    int64_t n_sparse;            /* number of sparse tiles */
    const void *values;          /* values blob, patch_pack_sizes bytes */
    const void *meta;            /* metadata blob (may be NULL when n_sparse == 0) */
    const patch_tile_desc *desc; /* Tn*Tk descriptors */
} patch_weight;

/*
 * patch_pack_sizes: byte sizes of the three blobs of a packed N x K weight
 * with n_sparse sparse tiles (host only, no device work):
 *   values = (T - n_sparse)*32768 + n_sparse*16384, meta = n_sparse*2048,
 *   desc = 16*T.
 * Errors: PATCH_ERR_SHAPE; PATCH_ERR_INVALID_ARG for n_sparse outside [0, T]
 * or a NULL output pointer.
 */
PATCH_API patch_status_t patch_pack_sizes(int64_t N, int64_t K, int64_t n_sparse, size_t *values_bytes,
                                size_t *meta_bytes, size_t *desc_bytes);

/*
 * patch_hard_mask: the inference-time hard form of the hybrid mask
 * ("Learnable Distributions": tile selection and pattern selection).
 *   bitmap[t]          = argmax(tile_logits[t][0..1])   (0 dense, 1 sparse)
 *   pat_id[n][g]       = argmax(pattern_logits[n][g][0..5])
 *   W_masked[n][k]     = W[n][k] if the tile is dense, or the tile is sparse
 *                        and k%4 is kept by pat_id[n][k/4]; else +0.0 (0x0000)
 * argmax takes the first maximum: a later entry wins only when strictly
 * greater, so ties go to the lowest index and a NaN never displaces an
 * earlier entry.  pat_id is written for every group, dense tiles included.
 *   W              bf16 [N][K]
 *   tile_logits    fp32 [Tn][Tk][2]
 *   pattern_logits fp32 [N][K/4][6]
 *   W_masked       bf16 [N][K], or NULL to skip
 *   bitmap         u8 [Tn][Tk];  pat_id  u8 [N][K/4]
 * Alignment: W, W_masked, pattern_logits 16 bytes.
 */
PATCH_API patch_status_t patch_hard_mask(const uint16_t *W, int64_t N, int64_t K, const float *tile_logits,
                               const float *pattern_logits, uint16_t *W_masked, uint8_t *bitmap,
                               uint8_t *pat_id, int32_t *dev_status, void *stream);

/*
 * patch_pack: build the packed format ("Core Mechanism": dense tiles kept
 * whole, sparse tiles stored as their 2 kept values per group of 4 plus the
 * 2-bit positions).  W may be masked or not: only kept positions of sparse
 * tiles are read, so both give identical blobs.  Two launches: a scan of the
 * bitmap that writes the descriptors, then one CTA per tile.
 *   W        bf16 [N][K]; bitmap u8 [Tn][Tk] (nonzero = sparse);
 *   pat_id   u8 [N][K/4] (read only inside sparse tiles);
 *   n_sparse must equal the number of nonzero bitmap entries: the kernel
 *   sets PATCH_DEV_COUNT and writes nothing past the blob sizes otherwise;
 *   values/meta/desc sized by patch_pack_sizes (meta may be NULL if n_sparse == 0).
 * An id > 5 in a sparse tile sets PATCH_DEV_BAD_PATTERN and is packed as id 0.
 */
PATCH_API patch_status_t patch_pack(const uint16_t *W, int64_t N, int64_t K, const uint8_t *bitmap,
                          const uint8_t *pat_id, int64_t n_sparse, void *values, void *meta,
                          patch_tile_desc *desc, int32_t *dev_status, void *stream);

/*
 * patch_soft_mask: the training-time (soft) form of the hybrid mask ("Core
 * Mechanism": a weighted combination of the dense and the 2:4 option;
 * "Learnable Distributions": tile and pattern choices sampled with
 * Gumbel-Softmax).  Per tile p = softmax((tile_logits + tile_noise) / tau) over
 * (dense, sparse); per group of 4 q = softmax((pattern_logits + pattern_noise)
 * / tau) over the 6 patterns; M[n][k] = p_dense + p_sparse * sum_j q_j
 * [k mod 4 in pattern j]; W_soft = W * M rounded once to bf16 (nearest even).
 * The pages give neither tau nor the noise: the Gumbel samples are the
 * caller's (NULL = no noise) and tau > 0 is an argument.  As tau -> 0 the
 * mask becomes patch_hard_mask's (pruned entries are then -0 for negative
 * weights: a product, not a select).  fp32 arithmetic with CUDA's expf.
 *   W bf16 [N][K]; tile_logits / tile_noise fp32 [Tn][Tk][2] (8-byte aligned);
 *   pattern_logits / pattern_noise fp32 [N][K/4][6]; W_soft bf16 [N][K] out;
 *   mask fp32 [N][K] out (nullable).  16-byte alignment otherwise.
 * Errors: PATCH_ERR_INVALID_ARG (NULL input, tau not positive and finite),
 * PATCH_ERR_SHAPE, PATCH_ERR_ALIGN, PATCH_ERR_DEVICE.
 */
PATCH_API patch_status_t patch_soft_mask(const uint16_t *W, int64_t N, int64_t K, const float *tile_logits,
                                         const float *tile_noise, const float *pattern_logits,
                                         const float *pattern_noise, float tau, uint16_t *W_soft, float *mask,
                                         void *stream);

/*
 * patch_hard_mask_tiles: patch_hard_mask with mask tiles of b x b, b =
 * mask_tile in {4, 8, 16, 32, 64, 128} ("Ablation Studies", tile size: the
 * learned tile can be as small as 4 x 4; hardware efficiency needs 128 x 128
 * execution tiles).  Same decisions and outputs as patch_hard_mask except
 *   tile_logits fp32 [N/b][K/b][2] (8-byte aligned), bitmap u8 [N/b][K/b],
 *   and W_masked[n][k] keeps W when tile (n/b, k/b) is dense.
 * mask_tile = 128 is patch_hard_mask.  To run a fine mask, pass its bitmap to
 * patch_exec_tiles and pack W_MASKED (not W) with the execution bitmap and
 * pat_id: dense execution tiles then carry the pruned zeros of their sparse
 * mask tiles, so the packed weight multiplies exactly as W_masked.
 * Errors: those of patch_hard_mask; PATCH_ERR_INVALID_ARG for another
 * mask_tile.
 */
PATCH_API patch_status_t patch_hard_mask_tiles(const uint16_t *W, int64_t N, int64_t K, int64_t mask_tile,
                                               const float *tile_logits, const float *pattern_logits,
                                               uint16_t *W_masked, uint8_t *bitmap, uint8_t *pat_id,
                                               int32_t *dev_status, void *stream);

/*
 * patch_exec_tiles: the 128 x 128 execution tiles of a b x b mask (b =
 * mask_tile, 4..128): exec[tn][tk] = 1 (2:4 sparse execution) only when all
 * (128/b)^2 mask tiles inside it are sparse, else 0 (dense execution).
 *   bitmap   u8 [N/b][K/b] (patch_hard_mask_tiles' output);
 *   exec     u8 [N/128][K/128] out, the bitmap patch_pack takes;
 *   n_sparse one int64 on the DEVICE out (8-byte aligned): the number of sparse
 *            execution tiles, for patch_pack_sizes.  It is zeroed on the stream
 *            and then counted, so it needs no initial value.
 * Errors: PATCH_ERR_INVALID_ARG (NULL, mask_tile), PATCH_ERR_SHAPE,
 * PATCH_ERR_ALIGN, PATCH_ERR_DEVICE.
 */
PATCH_API patch_status_t patch_exec_tiles(const uint8_t *bitmap, int64_t N, int64_t K, int64_t mask_tile,
                                          uint8_t *exec, int64_t *n_sparse, void *stream);

/*
 * patch_tile_kinds: the tile half of the hard mask alone ("Learnable
 * Distributions", item 1: a 2-way logit per tile chooses dense or 2:4 sparse).
 *   tile_logits fp32 [Tn][Tk][2] (index 0 = dense, 1 = sparse);
 *   bitmap      u8 [Tn][Tk] out: 1 where logit[1] > logit[0] (ties -> dense),
 *               the same decision patch_hard_mask takes;
 *   n_sparse    one int64 on the DEVICE out: the number of sparse tiles (the
 *               caller reads it to size the packed blobs with patch_pack_sizes).
 * The count is zeroed on the stream, then one launch fills both; no other
 * memory is touched.  Errors: PATCH_ERR_INVALID_ARG (NULL),
 * PATCH_ERR_SHAPE, PATCH_ERR_ALIGN (tile_logits or n_sparse not 8-byte aligned),
 * PATCH_ERR_DEVICE.
 */
PATCH_API patch_status_t patch_tile_kinds(const float *tile_logits, int64_t N, int64_t K, uint8_t *bitmap,
                                          int64_t *n_sparse, void *stream);

/*
 * patch_pack_from_logits: hard mask and pack in one pass, without the masked
 * weight or the pattern ids in memory.  Same output as patch_hard_mask
 * followed by patch_pack: every sparse tile's pattern ids are the argmax of
 * its 6 pattern logits per group (first maximum wins, as in patch_hard_mask),
 * taken inside the pack kernel; the pattern logits of dense tiles are never
 * read.  (Frozen pattern ids, as in the paper's tile-only variant, go through
 * patch_pack with pat_id instead.)
 *   W bf16 [N][K]; bitmap u8 [Tn][Tk] (from patch_tile_kinds or patch_hard_mask);
 *   pattern_logits fp32 [N][K/4][6] (16-byte aligned); n_sparse, values,
 *   meta, desc, dev_status as for patch_pack (PATCH_DEV_COUNT on a count
 *   mismatch, nothing written past the blob sizes).
 */
PATCH_API patch_status_t patch_pack_from_logits(const uint16_t *W, int64_t N, int64_t K, const uint8_t *bitmap,
                                                const float *pattern_logits, int64_t n_sparse, void *values,
                                                void *meta, patch_tile_desc *desc, int32_t *dev_status,
                                                void *stream);

/*
 * patch_gemm_workspace_size: device scratch bytes patch_gemm needs for M rows
 * of X and this weight, enough for every path M can take (0 when none is
 * needed: the prefill path at an M that fills the GPU).  Host only, but
 * queries the current device's SM count.
 */
PATCH_API patch_status_t patch_gemm_workspace_size(int64_t M, const patch_weight *W, size_t *bytes);

/*
 * patch_gemm: Y = X * W_eff^T with fp32 accumulation and one round to
 * bf16 (nearest-even) at the end ("Inference & Deployment": dense tiles on
 * the dense tensor-core MMA, sparse tiles on the 2:4 sparse tensor-core MMA).
 *   X  bf16 [M][K] (16-byte aligned, M >= 0; M == 0 is a no-op)
 *   W  packed weight (host struct)
 *   Y  bf16 [M][N] (16-byte aligned)
 *   workspace: patch_gemm_workspace_size bytes (may be NULL when that is 0).
 *     Its first 64 KiB hold the arrival counters of the decode path and of
 *     the prefill path's split-K mode: they must be zero before the first
 *     use, and every successful call leaves them zero; the rest is scratch
 *     (fp32 partial sums) whose contents do not matter.  So one zero-fill at
 *     allocation suffices, and one workspace of the largest size serves every
 *     layer, token count and path, in any order.  After a call that reported
 *     an error, zero it again.  The decode path needs it 16-byte aligned
 *     (PATCH_ERR_WORKSPACE otherwise); the prefill path uses it only when it
 *     is aligned and large enough for the split-K partials.
 *     The tensor-core decode path takes layers of up to 4096 tile rows
 *     (N <= 524288); PATCH_PATH_AUTO sends wider ones to the CUDA-core decode
 *     path.
 * M <= 16 runs the decode path: 1.5 CTAs per SM each stream an equal share
 * of the stored panels through a TMA ring (stream-K), the tensor cores reduce
 * them (N = 16 tokens, zero-padded); a tile row cut between CTAs is finished
 * by the last CTA to reach it, which adds the fp32 partials in the
 * workspace in CTA order (deterministic).
 * Larger M runs the prefill path (TMA-fed tcgen05 kernel: each CTA takes two
 * tile rows x up to 240 tokens at a time, dense and sparse MMAs into one TMEM
 * fp32 accumulator per tile row).  When those units would leave SMs idle
 * (few tile rows and few tokens) and the workspace holds the fp32 partials,
 * K is split across CTAs and the last part of each output block to finish
 * adds the parts in K order (deterministic); with a smaller or NULL
 * workspace the whole-K units run instead.
 * The kernels are launched with programmatic dependent launch: they read W,
 * its metadata and descriptors before the previous kernel in the stream has
 * completed, and X only after.  X may therefore be that kernel's output; the
 * packed weight must not be written by a kernel that allows an early launch
 * of its successor (patch_pack does not).
 * A bounded wait that runs out sets PATCH_DEV_TIMEOUT (Y is then undefined).
 */
PATCH_API patch_status_t patch_gemm(const uint16_t *X, int64_t M, const patch_weight *W, uint16_t *Y,
                          void *workspace, size_t workspace_bytes, int32_t *dev_status,
                          void *stream);

/*
 * patch_gemm_ex: patch_gemm with an explicit path (PATCH_PATH_*) and the
 * bounded-wait limit of the tensor-core kernels in microseconds (0 =
 * default, 2 s).  PATCH_PATH_DECODE and PATCH_PATH_DECODE_SIMT require
 * M <= 16.  PATCH_PATH_TEST_STALL is only accepted together with
 * PATCH_PATH_PREFILL.  patch_gemm_workspace_size covers every path.
 */
PATCH_API patch_status_t patch_gemm_ex(const uint16_t *X, int64_t M, const patch_weight *W, uint16_t *Y,
                             void *workspace, size_t workspace_bytes, int32_t *dev_status,
                             void *stream, int path, uint64_t wait_limit_us);

/*
 * patch_gemm_chain_workspace_size / patch_gemm_chain: a sequence of decode
 * GEMMs (each M <= 16 tokens), Y_j = X_j * W_j_eff^T, run by one persistent
 * launch per up to PATCH_CHAIN_MAX_CALLS calls ("Inference & Deployment":
 * the same hybrid execution as patch_gemm's decode path; running a model's
 * layers back to back is how the pages measure LLaMA-2 7B end to end,
 * "Experimental Results" -> "Speedup & Efficiency").
 *
 * A decode GEMM is bound by the bytes of its packed weight, but a separate
 * launch per layer also pays, per layer, the drain of the previous kernel,
 * the start of its own CTAs, the X load once its input is ready and the
 * finish of tile rows cut between CTAs, while the memory idles.  In a chain
 * every CTA (one per SM, all resident: cooperative launch) streams the
 * weight panels of call j+1 into its shared-memory ring while call j ends;
 * only X waits for the previous call.
 *
 *   calls[j].X  bf16 [M][K] device, 16-byte aligned
 *   calls[j].Y  bf16 [M][N] device, 16-byte aligned
 *   calls[j].W  packed weight (by value; its blobs are caller-owned device memory)
 *   calls[j].M  0..16 (0: the call is skipped)
 *   calls[j].after_previous
 *       nonzero: X_j may be written by earlier calls of the chain, so call j
 *       reads X_j only after every earlier call has completed (Y written and
 *       visible) -- the ordering of separate patch_gemm calls on one stream;
 *       0: X_j is ready when the chain starts, and call j may overlap earlier
 *       calls.  A call with after_previous == 0 must not write memory that an
 *       earlier call reads or writes.  The first call of a chain never waits.
 * Results equal patch_gemm's decode path (same tile kernels, same fp32 sum
 * order within a tile row; cut rows are added in CTA order): within the GEMM
 * tolerance of each other, deterministic run to run.
 * workspace: patch_gemm_chain_workspace_size bytes, 16-byte aligned, zero
 * before the first use.  Its first 64 KiB are the counter region of
 * patch_gemm's workspace (completion counters of the calls, then arrival
 * counters of their cut tile rows), which every successful call leaves
 * zero; so one zero-filled workspace of the largest size serves patch_gemm
 * and patch_gemm_chain in any order.  After an error, zero it again.  The
 * rest is scratch: fp32 partial sums and, per panel of every call, the tile
 * it belongs to (written by a small kernel launched first).
 * Calls are split into launches of at most PATCH_CHAIN_MAX_CALLS calls whose
 * tile rows fit the counter region (4 counters per tile row); each launch
 * starts after the previous one in the stream has completed.
 * Limits: N <= 524160 per call (4095 tile rows).  Every wait (on a ring
 * slot or on another CTA's completion counter) is bounded by wait_limit_us
 * (0 = 2 s); on expiry PATCH_DEV_TIMEOUT is set and Y is undefined.
 * Errors: PATCH_ERR_INVALID_ARG (NULL, M outside 0..16, n_calls < 0),
 * PATCH_ERR_SHAPE, PATCH_ERR_ALIGN, PATCH_ERR_WORKSPACE, PATCH_ERR_DEVICE,
 * PATCH_ERR_CUDA (including a GPU that cannot keep one CTA per SM resident).
 */
#define PATCH_CHAIN_MAX_CALLS 64
typedef struct {
    const uint16_t *X;
    uint16_t *Y;
    patch_weight W;
    int64_t M;
    int32_t after_previous;
    int32_t reserved; /* set to 0 */
} patch_chain_call;
PATCH_API patch_status_t patch_gemm_chain_workspace_size(const patch_chain_call *calls, int64_t n_calls,
                                                         size_t *bytes);
PATCH_API patch_status_t patch_gemm_chain(const patch_chain_call *calls, int64_t n_calls, void *workspace,
                                          size_t workspace_bytes, int32_t *dev_status, void *stream,
                                          uint64_t wait_limit_us);

/*
 * patch_gemm_group: independent GEMMs Y_j = X_j * W_j_eff^T, each with any
 * token count, run by one persistent launch of the prefill kernel per up to
 * PATCH_GROUP_MAX_CALLS calls ("Inference & Deployment": the same hybrid
 * execution as patch_gemm's prefill path: dense tiles on the dense
 * tensor-core MMA, sparse tiles on the 2:4 sparse one, fp32 accumulation in
 * tensor memory, one rounding to bf16).
 *
 * A prefill GEMM of few tile rows or few tokens (the projections of a small
 * model, or k and v beside q) has fewer units (2 tile rows x up to 240
 * tokens) than the GPU has SMs, and as its own kernel it also pays its
 * set-up, first loads and last partial wave.  Here the units of all the
 * calls share one grid: the host deals them out to the CTAs longest first
 * (work modelled as K-tiles x tokens x tile rows), each to the CTA with the
 * least work so far.  Token blocks are the fewest of at most 240 tokens,
 * evened out (M = 512: three of 176).
 *
 *   calls[j].X, .Y, .W, .M as for patch_gemm_chain, but M may be any value
 *       0 .. 2^30 (0: the call is skipped; M <= 16 runs in 16-token units on
 *       the tensor-core prefill kernel, where patch_gemm_chain is faster)
 *   calls[j].after_previous must be 0: the calls are independent, and no
 *       call may write memory that another call of the group reads or writes
 *   calls[j].reserved: ignored
 * No workspace: K is never split.  Results: within the GEMM tolerance of
 * patch_gemm's (the token blocking, and so the order in which each output's
 * fp32 partial sums add up, may differ), deterministic run to run.  Every
 * wait is bounded by wait_limit_us (0 = 2 s); on expiry PATCH_DEV_TIMEOUT is
 * set in *dev_status and the Y_j are undefined.
 * Errors: PATCH_ERR_INVALID_ARG (NULL, M outside 0..2^30, after_previous set,
 * n_calls < 0), PATCH_ERR_SHAPE, PATCH_ERR_ALIGN, PATCH_ERR_DEVICE,
 * PATCH_ERR_CUDA.
 */
#define PATCH_GROUP_MAX_CALLS 32
PATCH_API patch_status_t patch_gemm_group(const patch_chain_call *calls, int64_t n_calls, int32_t *dev_status,
                                          void *stream, uint64_t wait_limit_us);

/*
 * patch_gemm_decode_noalloc: the decode GEMM (M <= 16) for callers that
 * cannot allocate device memory.  The paper has no counterpart; this is a
 * deployment convenience of this library.
 *
 * Some callers have no way to get scratch memory: a plugin inside a host
 * framework that owns the device memory pool and passes the plugin only its
 * input and output buffers, or a latency-critical loop where a cudaMalloc
 * (which may synchronise the whole device) is not acceptable.  This entry
 * point runs the CUDA-core split-K decode path (the one patch_gemm_ex runs
 * with PATCH_PATH_DECODE_SIMT), not patch_gemm's default tensor-core decode
 * kernel, and keeps that path's split-K partial sums in a buffer compiled
 * into the library instead of a caller-provided workspace.  Its output
 * therefore equals patch_gemm's within the GEMM tolerance (relative
 * Frobenius error <= 5e-3, |err| <= 1e-2 (1 + |ref|)), not bit for bit: the
 * two paths add the fp32 products in different orders.
 *   - the buffer is PATCH_NOALLOC_SCRATCH_BYTES of device memory that every
 *     GPU which loads the library holds until the process exits;
 *   - the first call on each device looks the buffer's device address up
 *     (cudaGetSymbolAddress, with that device current), so make that first
 *     call before any stream capture;
 *   - a problem whose partial sums need more than the buffer holds is
 *     rejected with PATCH_ERR_WORKSPACE (no launch); the partials take
 *     S * M * N * 4 bytes, S being the number of K splits the path chooses
 *     (1, needing none, when the layer alone has enough row slabs to fill
 *     the GPU);
 *   - every call shares the one buffer: calls whose kernels may overlap on
 *     the GPU (different streams, or different host threads) race and give
 *     wrong results; serialise them, e.g. on one stream.  Nothing in the
 *     buffer needs to start at zero: each call overwrites what it reads.
 * X, Y and the packed weight are caller-owned device memory as for
 * patch_gemm; M must be in 0..16.  This path has no bounded waits and checks
 * no pattern ids, so it never sets a device status bit: dev_status is
 * accepted for symmetry with patch_gemm and may be NULL.  The call allocates
 * nothing and never synchronises the stream.
 */
#define PATCH_NOALLOC_SCRATCH_BYTES (4u << 20) /* 4 MiB */
PATCH_API patch_status_t patch_gemm_decode_noalloc(const uint16_t *X, int64_t M, const patch_weight *W,
                                                   uint16_t *Y, int32_t *dev_status, void *stream);

/*
 * patch_gemm_mlp_workspace_size / patch_gemm_mlp: the first half of LLaMA's
 * gated MLP on two hybrid weights of the same shape,
 *   H[m][n] = silu(G[m][n]) * U[m][n],  G = X W_gate_eff^T,  U = X W_up_eff^T,
 * silu(z) = z / (1 + e^-z), fp32 accumulation, one round to bf16 at the end
 * (the linears of the pages' LLaMA-2 7B end-to-end runs, "Experimental
 * Results" -> "Speedup & Efficiency"; the gated SiLU is LLaMA's, not stated
 * by the pages).
 *   X bf16 [M][K]; W_gate, W_up packed [N][K] each; H bf16 [M][N] (16-byte aligned).
 * M > 16: one prefill launch in which each unit multiplies a gate tile row and
 * the up tile row of the same 128 features against the same X panels and the
 * epilogue writes H directly (G and U never reach memory).
 * M <= 16: two decode GEMMs write G and U (bf16) into the workspace, then one
 * elementwise launch forms H.
 * workspace: patch_gemm_mlp_workspace_size bytes, zero-filled before its first
 * use: a patch_gemm workspace (whose counter region every successful call
 * leaves zero) followed by G and U.
 * Errors as patch_gemm; PATCH_ERR_SHAPE also when the two weights differ in shape.
 */
PATCH_API patch_status_t patch_gemm_mlp_workspace_size(int64_t M, const patch_weight *W_gate, const patch_weight *W_up,
                                                       size_t *bytes);
PATCH_API patch_status_t patch_gemm_mlp(const uint16_t *X, int64_t M, const patch_weight *W_gate,
                                        const patch_weight *W_up, uint16_t *H, void *workspace, size_t workspace_bytes,
                                        int32_t *dev_status, void *stream);

/*
 * patch_shard_rows: column-parallel split of one layer over n_shards GPUs
 * (output features are independent, so each GPU multiplies a contiguous range
 * of tile rows and the full Y is the concatenation of the shards' Y along N).
 * Balanced by stored bytes, not by rows: tile row r stores
 *   bytes(r) = sum over its Tk tiles of (dense ? 32768 : 18432) + 16 * Tk,
 * and shard i (0-based) is [row_begin[i], row_begin[i + 1]) where
 * row_begin[0] = 0, row_begin[n_shards] = Tn and, for 0 < i < n_shards,
 * row_begin[i] is the first row whose prefix sum of bytes (rows before it)
 * reaches i / n_shards of the total, then moved, if needed, to keep every
 * shard non-empty (row_begin[i - 1] < row_begin[i] <= Tn - (n_shards - i)).
 *   bitmap    HOST u8 [Tn][Tk] (nonzero = sparse);
 *   row_begin HOST int64 [n_shards + 1] out.
 * Host only, no device work.  Errors: PATCH_ERR_INVALID_ARG (NULL, Tn or Tk < 1,
 * n_shards < 1 or > Tn).
 */
PATCH_API patch_status_t patch_shard_rows(const uint8_t *bitmap, int64_t Tn, int64_t Tk, int64_t n_shards,
                                          int64_t *row_begin);

/*
 * patch_shard_rows_by: patch_shard_rows with a choice of what the shards
 * balance (the same prefix rule and the same non-empty adjustment):
 *   by = PATCH_SHARD_BY_BYTES: the stored bytes above (decode, M <= 16, streams
 *        them: patch_shard_rows itself);
 *   by = PATCH_SHARD_BY_FLOPS: the tensor cores' work, 2 per dense tile and 1
 *        per sparse tile (prefill: a sparse tile's MMAs multiply half of W,
 *        "Inference & Deployment"), so that each GPU's prefill GEMM takes the
 *        same time rather than moving the same bytes.
 * Host only.  Errors as patch_shard_rows, and PATCH_ERR_INVALID_ARG for any
 * other value of by.
 */
#define PATCH_SHARD_BY_BYTES 0
#define PATCH_SHARD_BY_FLOPS 1
PATCH_API patch_status_t patch_shard_rows_by(const uint8_t *bitmap, int64_t Tn, int64_t Tk, int64_t n_shards,
                                             int64_t by, int64_t *row_begin);

/*
 * patch_mma_probe: a measurement of this GPU's tensor-core MMA rate for the
 * two instruction forms of the hybrid GEMM ("Inference & Deployment": dense
 * tiles on the dense tensor-core MMA, sparse tiles on the 2:4 sparse one),
 * free of memory traffic: one CTA per SM issues `iters` rounds of four
 * M = 128, N = 240 MMAs (the prefill kernel's shape) on pseudo-random bf16
 * operands in shared memory.  A dense round is four K = 16 MMAs, a sparse
 * round four K = 32 (logical) .sp MMAs with valid metadata, so a round does
 * 4 x 2 x 128 x 240 x 16 (dense) or x 32 (sparse, dense-equivalent) FLOPs on
 * each SM.  The caller times the launch on `stream` (the call itself never
 * synchronises); the ratio of the two rates is the sparse/dense speed ratio
 * that the prefill path's mixed roofline needs.  dev_status gets
 * PATCH_DEV_TIMEOUT if the final wait for the MMAs runs out (2 s).
 * Errors: PATCH_ERR_INVALID_ARG (iters < 1, NULL dev_status), PATCH_ERR_DEVICE,
 * PATCH_ERR_CUDA.
 */
PATCH_API patch_status_t patch_mma_probe(int sparse, int64_t iters, int32_t *dev_status, void *stream);

/*
 * patch_check_weight: check a packed weight's descriptor table against the
 * packed format on the device ("Core Mechanism": dense tiles whole, 2:4 tiles
 * as their kept half): every tile's kind is 0 or 1, a sparse tile's ordinal
 * counts the sparse tiles before it (a dense tile's is 0xFFFFFFFF), every
 * values offset is the sum of the sizes of the tiles before it, and the table
 * holds exactly n_sparse sparse tiles.  A weight that passes only indexes
 * memory inside its blobs in every GEMM path.  A violation ORs
 * PATCH_DEV_BOUNDS into *dev_status (read it with patch_read_status).  One
 * launch of one CTA on `stream`; reads only the Tn*Tk descriptors.  Use it on
 * weights that did not come from patch_pack in this process (loaded from a
 * file, received from elsewhere).
 *
 * Debug build.  The library can also be built with PATCH_DEBUG defined
 * (libpatch_debug.so: `python -m tile_sparse_gemm_b200.build --debug`).  There
 * every GEMM entry point (patch_gemm, patch_gemm_ex, patch_gemm_mlp,
 * patch_gemm_chain, patch_gemm_decode_noalloc) first runs this check on each
 * weight it is given, synchronises the stream, and returns PATCH_ERR_BOUNDS
 * without launching the GEMM when a weight fails; the GEMM kernels then only
 * see indices inside the weight's blobs.  The debug build therefore
 * synchronises in those calls (it cannot be captured in a CUDA graph), and
 * patch_gemm_decode_noalloc needs a non-NULL dev_status there.
 * Errors: PATCH_ERR_INVALID_ARG (NULL), PATCH_ERR_SHAPE, PATCH_ERR_ALIGN,
 * PATCH_ERR_DEVICE, PATCH_ERR_CUDA.
 */
PATCH_API patch_status_t patch_check_weight(const patch_weight *W, int32_t *dev_status, void *stream);

/*
 * ---- 64 x 64 execution tiles ("Experimental Results", "Ablation Studies",
 * tile size: finer tiles give more control over where the 2:4 pattern
 * applies, and with 128 x 128 masks every tile still runs on the hardware's
 * efficient path).  A second packed format that executes 64 x 64 tiles, with
 * its own calls, so that a mask of 64 x 64 tiles (or finer) keeps every
 * sparse 64-tile sparse instead of only the 128-tiles whose four quarters
 * are all sparse.  The hybrid layer it computes is the same; the GEMM runs
 * M = 64 tensor-core MMAs (dense kind::f16 K = 16, and the 2:4 sparse form
 * K = 32), which this GPU executes at half the FLOP rate of the M = 128
 * forms for dense tiles (patch_mma_probe_m measures both).
 *
 * Format (this library's specification):
 *   - Tiles of 64 x 64 in row-major tile order t = tn*(K/64) + tk; N and K
 *     multiples of 64.  Descriptors as for the 128 x 128 format
 *     (patch_tile_desc: kind, sparse ordinal, byte offset of the first panel).
 *   - Values blob: panels of 64 rows x 32 bf16, row major with 64-byte rows
 *     (4096 bytes).  A dense tile occupies 2 panels (the tile's k 0..31, then
 *     k 32..63); a sparse tile 1 panel in which row r holds, for each group
 *     g = 0..15, its two kept values in ascending k at positions 2g, 2g+1.
 *   - Metadata blob: 512 bytes per sparse tile at sparse_ordinal*512.  Group
 *     g of row r has the 4-bit code i0 | (i1 << 2) in the low nibble of its
 *     byte when g is even, the high nibble when g is odd; the byte is
 *         ((g>>1)&1) | ((r>>3)&1)<<1 | (g>>3)<<2 | (r&7)<<3
 *         | ((g>>2)&1)<<6 | (r>>4)<<7.
 *     This is the tensor-memory placement the 16-bit sparse MMA with M = 64
 *     reads (rows 16q..16q+15 in the first 16 lanes of lane quarter q, one
 *     32-bit column per K = 32 step), stored 8 bytes per lane so that each
 *     quarter's 128 bytes move with one 32-lane, 2-column tensor-memory store.
 *   - All blobs 16-byte aligned.
 */
#define PATCH_TILE64 64
#define PATCH_PANEL64_BYTES 4096
#define PATCH_DENSE_TILE64_BYTES 8192
#define PATCH_SPARSE_TILE64_BYTES 4096
#define PATCH_META_TILE64_BYTES 512

/* A weight packed in the 64 x 64 format (host struct of device pointers, owned by the caller). */
typedef struct {
    int64_t N, K;                /* logical shape of W (multiples of 64) */
    int64_t n_sparse;            /* number of sparse 64 x 64 tiles */
    const void *values;          /* values blob, patch_pack64_sizes bytes */
    const void *meta;            /* metadata blob (may be NULL when n_sparse == 0) */
    const patch_tile_desc *desc; /* (N/64)*(K/64) descriptors */
} patch_weight64;

/*
 * patch_pack64_sizes: blob sizes of the 64 x 64 format (host only):
 *   values = (T - n_sparse)*8192 + n_sparse*4096, meta = n_sparse*512,
 *   desc = 16*T with T = (N/64)*(K/64).
 * Errors: PATCH_ERR_SHAPE (N, K not positive multiples of 64, or > 2^31);
 * PATCH_ERR_INVALID_ARG (n_sparse outside [0, T], NULL output).
 */
PATCH_API patch_status_t patch_pack64_sizes(int64_t N, int64_t K, int64_t n_sparse, size_t *values_bytes,
                                            size_t *meta_bytes, size_t *desc_bytes);

/*
 * patch_exec_tiles64: the 64 x 64 execution tiles of a b x b mask (b =
 * mask_tile in {4, 8, 16, 32, 64}): exec[tn][tk] = 1 only when all (64/b)^2
 * mask tiles inside it are sparse (at b = 64 the bitmap itself).
 *   bitmap u8 [N/b][K/b]; exec u8 [N/64][K/64] out; n_sparse one int64 on the
 *   DEVICE out (8-byte aligned), zeroed on the stream and then counted.
 * Errors: PATCH_ERR_INVALID_ARG (NULL, mask_tile), PATCH_ERR_SHAPE,
 * PATCH_ERR_ALIGN, PATCH_ERR_DEVICE, PATCH_ERR_CUDA.
 */
PATCH_API patch_status_t patch_exec_tiles64(const uint8_t *bitmap, int64_t N, int64_t K, int64_t mask_tile,
                                            uint8_t *exec, int64_t *n_sparse, void *stream);

/*
 * patch_pack64: build the 64 x 64 format from W, an execution bitmap
 * [N/64][K/64] (nonzero = sparse) and pattern ids u8 [N][K/4] (read only in
 * sparse tiles).  As for patch_pack: only kept positions of sparse tiles are
 * read (W masked or not gives the same blobs); n_sparse must equal the
 * bitmap's count (PATCH_DEV_COUNT otherwise, nothing written past the blob
 * sizes); an id > 5 sets PATCH_DEV_BAD_PATTERN and is packed as id 0.
 * values/meta/desc sized by patch_pack64_sizes.  Two launches (scan, tiles).
 * Errors: PATCH_ERR_INVALID_ARG, PATCH_ERR_SHAPE, PATCH_ERR_ALIGN (W, blobs
 * 16-byte aligned), PATCH_ERR_DEVICE, PATCH_ERR_CUDA.
 */
PATCH_API patch_status_t patch_pack64(const uint16_t *W, int64_t N, int64_t K, const uint8_t *bitmap,
                                      const uint8_t *pat_id, int64_t n_sparse, void *values, void *meta,
                                      patch_tile_desc *desc, int32_t *dev_status, void *stream);

/*
 * patch_gemm64_workspace_size: device scratch bytes patch_gemm64 needs for M
 * rows of X and this weight (host only; queries the SM count).
 */
PATCH_API patch_status_t patch_gemm64_workspace_size(int64_t M, const patch_weight64 *W, size_t *bytes);

/*
 * patch_gemm64: Y = X * W_eff^T for a weight in the 64 x 64 format, fp32
 * accumulation in tensor memory and one round to bf16 (nearest even).
 *   X bf16 [M][K] (16-byte aligned, M >= 0; M == 0 is a no-op);
 *   Y bf16 [M][N];
 *   workspace: patch_gemm64_workspace_size bytes, 16-byte aligned.  Its
 *     first part holds arrival counters that must be zero before the first
 *     use and that every successful call leaves zero (zero it again after a
 *     call that reported an error); the rest is scratch.
 * One kernel: the tokens are cut into blocks of 16 (M <= 16; two CTAs per
 * SM) or 256 tokens (one CTA per SM), and the CTAs split the sequence of
 * (token block, tile) pairs into shares of equal stored bytes (stream-K).  A
 * CTA accumulates each tile row's tiles in tensor memory (M = 64 MMAs, N =
 * the token block); a tile row cut between CTAs is finished by the last
 * covering CTA, which adds the fp32 partials in CTA order (deterministic).
 * Sparse tiles' metadata goes from shared to tensor memory through
 * registers.  Launched with
 * programmatic dependent launch as patch_gemm (X may be the previous
 * kernel's output).  A bounded wait that runs out (wait_limit_us, 0 = 2 s)
 * sets PATCH_DEV_TIMEOUT.
 * Errors: PATCH_ERR_INVALID_ARG, PATCH_ERR_SHAPE, PATCH_ERR_ALIGN,
 * PATCH_ERR_WORKSPACE (too small or unaligned), PATCH_ERR_DEVICE,
 * PATCH_ERR_CUDA.
 */
PATCH_API patch_status_t patch_gemm64(const uint16_t *X, int64_t M, const patch_weight64 *W, uint16_t *Y,
                                      void *workspace, size_t workspace_bytes, int32_t *dev_status, void *stream,
                                      uint64_t wait_limit_us);

/*
 * patch_mma_probe_m: patch_mma_probe for MMA shape M = 64 or 128 (A of M
 * rows; same N = 240, K and rounds).  A round does 4 x 2 x M x 240 x 16
 * (dense) or x 32 (sparse) FLOPs per SM.  Errors as patch_mma_probe, and
 * PATCH_ERR_INVALID_ARG for another M.
 */
PATCH_API patch_status_t patch_mma_probe_m(int m, int sparse, int64_t iters, int32_t *dev_status, void *stream);

/*
 * patch_read_status: synchronise `stream`, copy *dev_status to *host_bits and
 * return the first error it encodes (PATCH_ERR_TIMEOUT, then BOUNDS, then
 * BAD_PATTERN, then COUNT) or PATCH_OK.  host_bits may be NULL.
 */
PATCH_API patch_status_t patch_read_status(const int32_t *dev_status, void *stream, int32_t *host_bits);

/* Static message for a status code. */
PATCH_API const char *patch_strerror(patch_status_t status);

/* Library version string. */
PATCH_API const char *patch_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PATCH_H */
