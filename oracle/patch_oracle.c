/*
 * CPU oracle for the PATCH hybrid tile-sparse linear layer Y = X * W^T.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check
 * and the benchmark's CPU-baseline leg may load this code.  It shares no
 * source, header, table or helper with the CUDA library: everything below is
 * written out again from the method's description and the packed-format
 * specification.  It is deliberately plain and slow: loops in the order the
 * definitions read, fp64 accumulation, no blocking or reordering.
 *
 * Method (PATCH: Learnable Tile-level Hybrid Sparsity for LLMs; page
 * "gist.science/paper/2509.23410", section 2 "Methodology: PATCH",
 * subsections "Core Mechanism" and "Learnable Distributions"):
 *   - W (N x K) is cut into equal tiles; each tile is either dense (0%
 *     sparsity) or 2:4 sparse (50% sparsity).  Execution tile: 128 x 128
 *     ("Inference & Deployment"; "Ablation Studies", tile size).
 *   - The hybrid mask combines a dense option and a 2:4 option per tile; the
 *     tile choice comes from a learnable 2-way logit distribution, and inside
 *     sparse tiles a separate learnable distribution picks one of the 6
 *     possible 2:4 patterns per group of 4.
 *   - At inference the mask is fixed: each choice is the argmax of its logits
 *     (reading: deterministic argmax, first maximum wins on ties, a NaN never
 *     beats an earlier value).
 *   - Groups of 4 run along K (4 consecutive input features of one W row).
 *   - Pattern ids: the kept pair (i0,i1), i0<i1, numbered in lexicographic
 *     order: 0:(0,1) 1:(0,2) 2:(0,3) 3:(1,2) 4:(1,3) 5:(2,3).
 *   - A pruned weight becomes +0.0 (bit pattern 0x0000).
 *
 * Packed format (the library's own specification; the pages fix no format):
 *   - Tiles in row-major tile order t = tn*Tk + tk.
 *   - Descriptor (16 bytes, little endian): u32 kind (0 dense, 1 sparse),
 *     u32 sparse ordinal (number of sparse tiles before t; 0xFFFFFFFF for a
 *     dense tile), u64 byte offset of the tile's payload in the values blob.
 *   - Values blob: a sequence of "panels", each 128 rows x 64 bf16 stored row
 *     major (128-byte rows, 16384 bytes).  A dense tile occupies 2 panels
 *     (k 0..63, then k 64..127 of the tile).  A sparse tile occupies 1 panel:
 *     row r holds, for each group g = 0..31, the two kept values in ascending
 *     k at positions 2g and 2g+1.
 *   - Metadata blob: 2048 bytes per sparse tile at ordinal*2048.  The 4-bit
 *     code of group g of tile row r is i0 | (i1 << 2); it sits in the low
 *     nibble of its byte when g is even and in the high nibble when g is odd,
 *     at byte
 *        ((g>>1)&1) | ((r>>3)&1)<<1 | (g>>3)<<2 | (r&7)<<4
 *        | ((g>>2)&1)<<7 | (r>>4)<<8 .
 *
 * Mask tiles smaller than 128 x 128 (oracle_hard_mask_tiles,
 * oracle_exec_tiles) follow "Ablation Studies" (tile size) with the reading
 * that the execution tile stays 128 x 128 and runs sparse only when all its
 * mask tiles are sparse.
 *
 * The 64 x 64 execution-tile format (oracle_*64, oracle_exec_tiles_e,
 * oracle_apply_mask_tiles) is described above its functions near the end.
 *
 * Parity pins (tests/test_oracle.py): brute force over the 6 patterns with
 * one-hot logits, argmax ties, the exactly-2-of-4 invariant, global sparsity
 * = 0.5 x sparse-tile fraction, all-dense == numpy dense matmul, all-sparse
 * == numpy matmul of the 2:4-masked W, one-hot X columns, linearity over
 * tiles, pack/unpack round trip and closed-form blob sizes.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define TILE 128

enum { OK = 0, ERR_SHAPE = 1, ERR_BAD_PATTERN = 2, ERR_COUNT = 3, ERR_ALLOC = 4 };

/* The 6 ways of keeping 2 of 4 positions, in lexicographic order. */
static const int KEEP[6][2] = {{0, 1}, {0, 2}, {0, 3}, {1, 2}, {1, 3}, {2, 3}};

static double bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int shape_ok(int64_t N, int64_t K)
{
    return N > 0 && K > 0 && N % TILE == 0 && K % TILE == 0;
}

/* Index of the first maximum; a later entry wins only when strictly greater. */
static int argmax_first(const float *v, int n)
{
    int best = 0;
    float bv = v[0];
    for (int j = 1; j < n; ++j) {
        if (v[j] > bv) {
            bv = v[j];
            best = j;
        }
    }
    return best;
}

/* Is position k of row n kept under (bitmap, pattern ids)? -1 on a bad id. */
static int kept(int64_t n, int64_t k, int64_t K, const uint8_t *bitmap, const uint8_t *pat_id)
{
    int64_t Tk = K / TILE;
    if (bitmap[(n / TILE) * Tk + k / TILE] == 0)
        return 1;                      /* dense tile keeps everything */
    int id = pat_id[n * (K / 4) + k / 4];
    if (id > 5)
        return -1;
    int pos = (int)(k % 4);
    return pos == KEEP[id][0] || pos == KEEP[id][1];
}

/* The hybrid mask applied to W: W_eff = W where kept, +0.0 elsewhere. */
int oracle_apply_mask(const uint16_t *W, int64_t N, int64_t K, const uint8_t *bitmap,
                      const uint8_t *pat_id, uint16_t *W_eff)
{
    if (!shape_ok(N, K))
        return ERR_SHAPE;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int keep = kept(n, k, K, bitmap, pat_id);
            if (keep < 0)
                return ERR_BAD_PATTERN;
            W_eff[n * K + k] = keep ? W[n * K + k] : (uint16_t)0x0000;
        }
    }
    return OK;
}

/* Hard mask: argmax of tile logits [Tn][Tk][2] and pattern logits [N][K/4][6],
 * then the mask applied to W (W_masked may be NULL). */
int oracle_hard_mask(const uint16_t *W, int64_t N, int64_t K, const float *tile_logits,
                     const float *pattern_logits, uint16_t *W_masked, uint8_t *bitmap,
                     uint8_t *pat_id)
{
    if (!shape_ok(N, K))
        return ERR_SHAPE;
    int64_t T = (N / TILE) * (K / TILE);
    for (int64_t t = 0; t < T; ++t)
        bitmap[t] = (uint8_t)argmax_first(tile_logits + 2 * t, 2);
    int64_t G = N * (K / 4);
    for (int64_t i = 0; i < G; ++i)
        pat_id[i] = (uint8_t)argmax_first(pattern_logits + 6 * i, 6);
    if (W_masked)
        return oracle_apply_mask(W, N, K, bitmap, pat_id, W_masked);
    return OK;
}

/*
 * Mask tiles smaller than the execution tile ("Ablation Studies", tile size:
 * the learned tile may be as small as 4 x 4, while hardware efficiency needs
 * 128 x 128 execution tiles).  The mask tile is b x b, b a power of two from
 * 4 to 128; tile logits are [N/b][K/b][2] and the bitmap [N/b][K/b].  Each
 * choice is the argmax as above; position k of row n is kept when its b x b
 * tile is dense, or when k mod 4 is in the pattern of its group.
 */
static int mask_tile_ok(int64_t b)
{
    return b == 4 || b == 8 || b == 16 || b == 32 || b == 64 || b == 128;
}

int oracle_hard_mask_tiles(const uint16_t *W, int64_t N, int64_t K, int64_t b, const float *tile_logits,
                           const float *pattern_logits, uint16_t *W_masked, uint8_t *bitmap,
                           uint8_t *pat_id)
{
    if (!shape_ok(N, K) || !mask_tile_ok(b))
        return ERR_SHAPE;
    int64_t Tnb = N / b, Tkb = K / b;
    for (int64_t t = 0; t < Tnb * Tkb; ++t)
        bitmap[t] = (uint8_t)argmax_first(tile_logits + 2 * t, 2);
    int64_t G = N * (K / 4);
    for (int64_t i = 0; i < G; ++i)
        pat_id[i] = (uint8_t)argmax_first(pattern_logits + 6 * i, 6);
    if (!W_masked)
        return OK;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int keep = 1;
            if (bitmap[(n / b) * Tkb + k / b]) {
                int id = pat_id[n * (K / 4) + k / 4];
                int pos = (int)(k % 4);
                keep = pos == KEEP[id][0] || pos == KEEP[id][1];
            }
            W_masked[n * K + k] = keep ? W[n * K + k] : (uint16_t)0x0000;
        }
    }
    return OK;
}

/*
 * Execution tiles of a b x b mask: the 128 x 128 execution tile (tn, tk) runs
 * on the 2:4 sparse path only when every mask tile inside it is sparse; any
 * dense mask tile makes it a dense execution tile (whose sparse mask tiles
 * then carry their pruned zeros explicitly).  Writes exec [N/128][K/128] and
 * returns the number of sparse execution tiles through *n_sparse.
 */
int oracle_exec_tiles(const uint8_t *bitmap, int64_t N, int64_t K, int64_t b, uint8_t *exec, int64_t *n_sparse)
{
    if (!shape_ok(N, K) || !mask_tile_ok(b))
        return ERR_SHAPE;
    int64_t Tn = N / TILE, Tk = K / TILE, Tkb = K / b, r = TILE / b;
    int64_t count = 0;
    for (int64_t tn = 0; tn < Tn; ++tn) {
        for (int64_t tk = 0; tk < Tk; ++tk) {
            int all_sparse = 1;
            for (int64_t i = 0; i < r; ++i)
                for (int64_t j = 0; j < r; ++j)
                    if (!bitmap[(tn * r + i) * Tkb + tk * r + j])
                        all_sparse = 0;
            exec[tn * Tk + tk] = (uint8_t)all_sparse;
            count += all_sparse;
        }
    }
    *n_sparse = count;
    return OK;
}

/* Byte of the metadata block that holds group g (0..31) of tile row r (0..127). */
static int64_t meta_byte(int r, int g)
{
    return (int64_t)(((g >> 1) & 1) | (((r >> 3) & 1) << 1) | ((g >> 3) << 2) | ((r & 7) << 4) |
                     (((g >> 2) & 1) << 7) | ((r >> 4) << 8));
}

static void put_u32(uint8_t *p, uint32_t v)
{
    for (int i = 0; i < 4; ++i)
        p[i] = (uint8_t)(v >> (8 * i));
}

static void put_u64(uint8_t *p, uint64_t v)
{
    for (int i = 0; i < 8; ++i)
        p[i] = (uint8_t)(v >> (8 * i));
}

static uint64_t get_u64(const uint8_t *p)
{
    uint64_t v = 0;
    for (int i = 7; i >= 0; --i)
        v = (v << 8) | p[i];
    return v;
}

static uint32_t get_u32(const uint8_t *p)
{
    return (uint32_t)p[0] | (uint32_t)p[1] << 8 | (uint32_t)p[2] << 16 | (uint32_t)p[3] << 24;
}

/* Blob sizes of the packed format. */
void oracle_pack_sizes(int64_t N, int64_t K, int64_t n_sparse, int64_t *values_bytes,
                       int64_t *meta_bytes, int64_t *desc_bytes)
{
    int64_t T = (N / TILE) * (K / TILE);
    *values_bytes = (T - n_sparse) * 32768 + n_sparse * 16384;
    *meta_bytes = n_sparse * 2048;
    *desc_bytes = T * 16;
}

/* Pack W under (bitmap, pattern ids) into values, metadata and descriptors. */
int oracle_pack(const uint16_t *W, int64_t N, int64_t K, const uint8_t *bitmap,
                const uint8_t *pat_id, int64_t n_sparse, uint8_t *values, uint8_t *meta,
                uint8_t *desc)
{
    if (!shape_ok(N, K))
        return ERR_SHAPE;
    int64_t Tn = N / TILE, Tk = K / TILE;
    int64_t counted = 0;
    for (int64_t t = 0; t < Tn * Tk; ++t)
        counted += bitmap[t] != 0;
    if (counted != n_sparse)
        return ERR_COUNT;
    memset(meta, 0, (size_t)(n_sparse * 2048));

    uint64_t offset = 0;
    uint32_t ordinal = 0;
    for (int64_t tn = 0; tn < Tn; ++tn) {
        for (int64_t tk = 0; tk < Tk; ++tk) {
            uint8_t *d = desc + 16 * (tn * Tk + tk);
            uint16_t *panel = (uint16_t *)(values + offset);
            int sparse = bitmap[tn * Tk + tk] != 0;
            put_u32(d, (uint32_t)sparse);
            put_u32(d + 4, sparse ? ordinal : 0xFFFFFFFFu);
            put_u64(d + 8, offset);
            if (!sparse) {
                for (int h = 0; h < 2; ++h)
                    for (int r = 0; r < TILE; ++r)
                        for (int c = 0; c < 64; ++c)
                            panel[h * TILE * 64 + r * 64 + c] =
                                W[(tn * TILE + r) * K + tk * TILE + h * 64 + c];
                offset += 32768;
            } else {
                uint8_t *mb = meta + (int64_t)ordinal * 2048;
                for (int r = 0; r < TILE; ++r) {
                    int64_t n = tn * TILE + r;
                    for (int g = 0; g < 32; ++g) {
                        int64_t k0 = tk * TILE + 4 * g;
                        int id = pat_id[n * (K / 4) + k0 / 4];
                        if (id > 5)
                            return ERR_BAD_PATTERN;
                        int i0 = KEEP[id][0], i1 = KEEP[id][1];
                        panel[r * 64 + 2 * g] = W[n * K + k0 + i0];
                        panel[r * 64 + 2 * g + 1] = W[n * K + k0 + i1];
                        uint8_t code = (uint8_t)(i0 | (i1 << 2));
                        mb[meta_byte(r, g)] |= (uint8_t)(code << (4 * (g & 1)));
                    }
                }
                offset += 16384;
                ordinal += 1;
            }
        }
    }
    return OK;
}

/* Rebuild the effective (masked) W from a packed blob, by its own decoding. */
int oracle_unpack(const uint8_t *values, const uint8_t *meta, const uint8_t *desc, int64_t N,
                  int64_t K, uint16_t *W_eff)
{
    if (!shape_ok(N, K))
        return ERR_SHAPE;
    int64_t Tn = N / TILE, Tk = K / TILE;
    for (int64_t tn = 0; tn < Tn; ++tn) {
        for (int64_t tk = 0; tk < Tk; ++tk) {
            const uint8_t *d = desc + 16 * (tn * Tk + tk);
            uint32_t kind = get_u32(d), ordinal = get_u32(d + 4);
            const uint16_t *panel = (const uint16_t *)(values + get_u64(d + 8));
            for (int r = 0; r < TILE; ++r) {
                int64_t n = tn * TILE + r;
                uint16_t *row = W_eff + n * K + tk * TILE;
                if (kind == 0) {
                    for (int c = 0; c < TILE; ++c)
                        row[c] = panel[(c / 64) * TILE * 64 + r * 64 + (c % 64)];
                } else {
                    const uint8_t *mb = meta + (int64_t)ordinal * 2048;
                    for (int g = 0; g < 32; ++g) {
                        int code = (mb[meta_byte(r, g)] >> (4 * (g & 1))) & 0xF;
                        int i0 = code & 3, i1 = code >> 2;
                        for (int i = 0; i < 4; ++i)
                            row[4 * g + i] = 0;
                        row[4 * g + i0] = panel[r * 64 + 2 * g];
                        row[4 * g + i1] = panel[r * 64 + 2 * g + 1];
                    }
                }
            }
        }
    }
    return OK;
}

/* Y[m][n] = sum_k X[m][k] * W_eff[n][k], fp64, one plain dot product per output,
 * for the listed rows m of X (rows == NULL: all M rows; Y row i <- X row rows[i]). */
int oracle_gemm_rows(const uint16_t *X, int64_t M, const int64_t *rows, int64_t n_rows,
                     const uint16_t *W_eff, int64_t N, int64_t K, double *Y)
{
    if (N <= 0 || K <= 0 || M < 0)
        return ERR_SHAPE;
    int64_t R = rows ? n_rows : M;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < R; ++i) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t m = rows ? rows[i] : i;
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k)
                s += bf16_to_double(X[m * K + k]) * bf16_to_double(W_eff[n * K + k]);
            Y[i * N + n] = s;
        }
    }
    return OK;
}

/* The whole layer: hybrid mask applied to W, then the fp64 matmul. */
int oracle_hybrid_gemm(const uint16_t *X, int64_t M, const int64_t *rows, int64_t n_rows,
                       const uint16_t *W, int64_t N, int64_t K, const uint8_t *bitmap,
                       const uint8_t *pat_id, double *Y)
{
    if (!shape_ok(N, K))
        return ERR_SHAPE;
    uint16_t *W_eff = (uint16_t *)malloc((size_t)(N * K) * sizeof(uint16_t));
    if (!W_eff)
        return ERR_ALLOC;
    int rc = oracle_apply_mask(W, N, K, bitmap, pat_id, W_eff);
    if (rc == OK)
        rc = oracle_gemm_rows(X, M, rows, n_rows, W_eff, N, K, Y);
    free(W_eff);
    return rc;
}

/*
 * 64 x 64 execution tiles ("Ablation Studies", tile size: smaller tiles give
 * finer control over where the 2:4 pattern applies; larger ones run more
 * efficiently on the hardware).  The library's second packed format runs the
 * same hybrid layer on 64 x 64 execution tiles:
 *   - Tiles 64 x 64 in row-major tile order t = tn*(K/64) + tk; N and K are
 *     multiples of 64.  Descriptors as in the 128 x 128 format.
 *   - Values blob: "panels" of 64 rows x 32 bf16 stored row major (64-byte
 *     rows, 4096 bytes).  A dense tile occupies 2 panels (k 0..31, then
 *     k 32..63); a sparse tile 1 panel in which row r holds, for each group
 *     g = 0..15, its two kept values in ascending k at positions 2g, 2g+1.
 *   - Metadata blob: 512 bytes per sparse tile at ordinal*512; the 4-bit
 *     code of group g of tile row r sits in nibble (g & 1) of byte
 *        ((g>>1)&1) | ((r>>3)&1)<<1 | (g>>3)<<2 | (r&7)<<3
 *        | ((g>>2)&1)<<6 | (r>>4)<<7 .
 * Mask tiles b x b with b <= E (E = 64 or 128) map to execution tiles by the
 * same rule as for 128: an execution tile is sparse only when every mask
 * tile inside it is sparse.
 */
#define TILE64 64

static int shape64_ok(int64_t N, int64_t K)
{
    return N > 0 && K > 0 && N % TILE64 == 0 && K % TILE64 == 0;
}

/* The hybrid mask with b x b tiles applied to W (b = 4..128, N and K multiples of b). */
int oracle_apply_mask_tiles(const uint16_t *W, int64_t N, int64_t K, int64_t b, const uint8_t *bitmap,
                            const uint8_t *pat_id, uint16_t *W_eff)
{
    if (!mask_tile_ok(b) || N <= 0 || K <= 0 || N % b != 0 || K % b != 0)
        return ERR_SHAPE;
    int64_t Tkb = K / b;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int keep = 1;
            if (bitmap[(n / b) * Tkb + k / b]) {
                int id = pat_id[n * (K / 4) + k / 4];
                if (id > 5)
                    return ERR_BAD_PATTERN;
                int pos = (int)(k % 4);
                keep = pos == KEEP[id][0] || pos == KEEP[id][1];
            }
            W_eff[n * K + k] = keep ? W[n * K + k] : (uint16_t)0x0000;
        }
    }
    return OK;
}

/* Execution tiles of size E (64 or 128) of a b x b mask bitmap (b <= E):
 * exec [N/E][K/E], sparse only when all its mask tiles are sparse. */
int oracle_exec_tiles_e(const uint8_t *bitmap, int64_t N, int64_t K, int64_t b, int64_t E, uint8_t *exec,
                        int64_t *n_sparse)
{
    if ((E != 64 && E != 128) || !mask_tile_ok(b) || b > E || N <= 0 || K <= 0 || N % E != 0 ||
        K % E != 0)
        return ERR_SHAPE;
    int64_t Tn = N / E, Tk = K / E, Tkb = K / b, r = E / b;
    int64_t count = 0;
    for (int64_t tn = 0; tn < Tn; ++tn) {
        for (int64_t tk = 0; tk < Tk; ++tk) {
            int all_sparse = 1;
            for (int64_t i = 0; i < r; ++i)
                for (int64_t j = 0; j < r; ++j)
                    if (!bitmap[(tn * r + i) * Tkb + tk * r + j])
                        all_sparse = 0;
            exec[tn * Tk + tk] = (uint8_t)all_sparse;
            count += all_sparse;
        }
    }
    *n_sparse = count;
    return OK;
}

/* Byte of a 64 x 64 tile's 512-byte metadata block that holds group g (0..15) of row r (0..63). */
static int64_t meta64_byte(int r, int g)
{
    return (int64_t)(((g >> 1) & 1) | (((r >> 3) & 1) << 1) | ((g >> 3) << 2) | ((r & 7) << 3) |
                     (((g >> 2) & 1) << 6) | ((r >> 4) << 7));
}

void oracle_pack64_sizes(int64_t N, int64_t K, int64_t n_sparse, int64_t *values_bytes, int64_t *meta_bytes,
                         int64_t *desc_bytes)
{
    int64_t T = (N / TILE64) * (K / TILE64);
    *values_bytes = (T - n_sparse) * 8192 + n_sparse * 4096;
    *meta_bytes = n_sparse * 512;
    *desc_bytes = T * 16;
}

/* Pack W into the 64 x 64 format under an execution bitmap [N/64][K/64] and pattern ids. */
int oracle_pack64(const uint16_t *W, int64_t N, int64_t K, const uint8_t *bitmap, const uint8_t *pat_id,
                  int64_t n_sparse, uint8_t *values, uint8_t *meta, uint8_t *desc)
{
    if (!shape64_ok(N, K))
        return ERR_SHAPE;
    int64_t Tn = N / TILE64, Tk = K / TILE64;
    int64_t counted = 0;
    for (int64_t t = 0; t < Tn * Tk; ++t)
        counted += bitmap[t] != 0;
    if (counted != n_sparse)
        return ERR_COUNT;
    memset(meta, 0, (size_t)(n_sparse * 512));

    uint64_t offset = 0;
    uint32_t ordinal = 0;
    for (int64_t tn = 0; tn < Tn; ++tn) {
        for (int64_t tk = 0; tk < Tk; ++tk) {
            uint8_t *d = desc + 16 * (tn * Tk + tk);
            uint16_t *panel = (uint16_t *)(values + offset);
            int sparse = bitmap[tn * Tk + tk] != 0;
            put_u32(d, (uint32_t)sparse);
            put_u32(d + 4, sparse ? ordinal : 0xFFFFFFFFu);
            put_u64(d + 8, offset);
            if (!sparse) {
                for (int h = 0; h < 2; ++h)
                    for (int r = 0; r < TILE64; ++r)
                        for (int c = 0; c < 32; ++c)
                            panel[h * TILE64 * 32 + r * 32 + c] =
                                W[(tn * TILE64 + r) * K + tk * TILE64 + h * 32 + c];
                offset += 8192;
            } else {
                uint8_t *mb = meta + (int64_t)ordinal * 512;
                for (int r = 0; r < TILE64; ++r) {
                    int64_t n = tn * TILE64 + r;
                    for (int g = 0; g < 16; ++g) {
                        int64_t k0 = tk * TILE64 + 4 * g;
                        int id = pat_id[n * (K / 4) + k0 / 4];
                        if (id > 5)
                            return ERR_BAD_PATTERN;
                        int i0 = KEEP[id][0], i1 = KEEP[id][1];
                        panel[r * 32 + 2 * g] = W[n * K + k0 + i0];
                        panel[r * 32 + 2 * g + 1] = W[n * K + k0 + i1];
                        uint8_t code = (uint8_t)(i0 | (i1 << 2));
                        mb[meta64_byte(r, g)] |= (uint8_t)(code << (4 * (g & 1)));
                    }
                }
                offset += 4096;
                ordinal += 1;
            }
        }
    }
    return OK;
}

/* Rebuild the effective W from a 64 x 64 packed blob, by its own decoding. */
int oracle_unpack64(const uint8_t *values, const uint8_t *meta, const uint8_t *desc, int64_t N, int64_t K,
                    uint16_t *W_eff)
{
    if (!shape64_ok(N, K))
        return ERR_SHAPE;
    int64_t Tn = N / TILE64, Tk = K / TILE64;
    for (int64_t tn = 0; tn < Tn; ++tn) {
        for (int64_t tk = 0; tk < Tk; ++tk) {
            const uint8_t *d = desc + 16 * (tn * Tk + tk);
            uint32_t kind = get_u32(d), ordinal = get_u32(d + 4);
            const uint16_t *panel = (const uint16_t *)(values + get_u64(d + 8));
            for (int r = 0; r < TILE64; ++r) {
                int64_t n = tn * TILE64 + r;
                uint16_t *row = W_eff + n * K + tk * TILE64;
                if (kind == 0) {
                    for (int c = 0; c < TILE64; ++c)
                        row[c] = panel[(c / 32) * TILE64 * 32 + r * 32 + (c % 32)];
                } else {
                    const uint8_t *mb = meta + (int64_t)ordinal * 512;
                    for (int g = 0; g < 16; ++g) {
                        int code = (mb[meta64_byte(r, g)] >> (4 * (g & 1))) & 0xF;
                        int i0 = code & 3, i1 = code >> 2;
                        for (int i = 0; i < 4; ++i)
                            row[4 * g + i] = 0;
                        row[4 * g + i0] = panel[r * 32 + 2 * g];
                        row[4 * g + i1] = panel[r * 32 + 2 * g + 1];
                    }
                }
            }
        }
    }
    return OK;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads for the following calls (the timing of the CPU baseline only). */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    omp_set_num_threads(n);
#else
    (void)n;
#endif
}
