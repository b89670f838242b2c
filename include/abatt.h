/*
 * abatt.h -- C ABI of the AB-Attention hot path on B200 (sm_100a).
 *
 * Method: "Accurate Block Attention (AB-Attention)", abstract.  Dynamic
 * block-sparse attention for video diffusion transformers in three stages:
 *   IBCS  the queries of each query block are clustered on their own (no
 *         token reordering) and the centroids estimate how much attention
 *         mass every key/value block receives;
 *   SIP   key/value blocks are drawn with probability proportional to those
 *         estimates and re-weighted by 1/(inclusion probability), so that one
 *         pass estimates dense attention instead of truncating it;
 *   gather kernel: the drawn key/value blocks (much smaller than a tile) are
 *         packed into full tensor-core tiles.
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers on the current CUDA device.
 *     The caller owns every buffer; the library never allocates or frees
 *     memory and keeps no state between calls other than cached kernel
 *     attributes.
 *   - Q, K, V, O: bf16, 16-byte aligned base, contiguous in the layout
 *     cfg->layout names: [B][H][N][d] (ABATT_LAYOUT_BHND, the default) or
 *     [B][N][H][d] (ABATT_LAYOUT_BNHD).  lse is [B][H][N] in both.
 *   - A "row" is one query block (beta, h, i), linear id
 *     ((beta*H)+h)*nQ + i, with nQ = ceil(N/q_block), nK = ceil(N/kv_block).
 *     The last query block and the last key block may be partial; missing
 *     rows/keys do not exist (masked from every softmax, never stored).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call is asynchronous on that stream.
 *   - Errors found on the host return immediately, before any launch.
 *     Errors found on the device (list overflow, a bounded wait that ran
 *     out) are OR-ed as ABATT_DEVFLAG_* bits into the 32-bit status word at
 *     the start of the call's workspace; read it with abatt_read_status.
 *     Nothing traps or spins without bound on the device.
 *   - Limits: d in {64, 128}; q_block == 128; kv_block in {16, 32, 64, 128};
 *     1 <= clusters <= 16; 0 <= kmeans_iters <= 64; nK <= 32767;
 *     B*H*nQ < 2^31.
 */
#ifndef ABATT_H
#define ABATT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum abatt_status {
    ABATT_OK = 0,
    ABATT_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad budget */
    ABATT_ERR_UNSUPPORTED = 2, /* a limit above is exceeded */
    ABATT_ERR_ALIGNMENT = 3,   /* a tensor base is not 16-byte aligned */
    ABATT_ERR_WORKSPACE = 4,   /* workspace missing or smaller than required */
    ABATT_ERR_CUDA = 5,        /* a CUDA runtime call failed */
    ABATT_ERR_CAPACITY = 6,    /* (device) a row drew more blocks than capacity */
    ABATT_ERR_TIMEOUT = 7,     /* (device) a bounded wait ran out */
    ABATT_ERR_DEVICE = 8       /* device status word holds an error */
} abatt_status;

/* Bits of the device status word. */
#define ABATT_DEVFLAG_CAPACITY 0x1u
#define ABATT_DEVFLAG_TIMEOUT 0x2u
#define ABATT_DEVFLAG_BADLIST 0x4u /* a block index outside [0, nK) was skipped */

typedef struct abatt_shape {
    int B; /* batch */
    int H; /* heads */
    int N; /* tokens (the flattened latent video grid, raster order) */
    int d; /* head dimension */
} abatt_shape;

/* How abatt_sample (and abatt_forward) turn block probabilities into lists.
   SIP: the abstract's sampler -- a Poisson draw with pi_b = min(1, c*p_b),
        sum pi = M, each drawn block weighted by 1/pi_b (log-weight -ln pi_b).
   TOPK: the truncating baseline the abstract contrasts it with -- the M blocks
        with the largest estimate (ranked on the same 48-bit fixed point, ties to
        the lower index), each with log-weight 0.  Needs nK <= 10240
        (ABATT_ERR_UNSUPPORTED otherwise). */
enum { ABATT_SELECT_SIP = 0, ABATT_SELECT_TOPK = 1 };

/* Where the sampler's uniforms come from.
   INDEPENDENT: Philox counter (b/4, i, h, beta) -- every query block draws on
        its own (the method as read).
   PAIRED: counter (b/4, floor(i/2), h, beta) -- query blocks 2j and 2j+1 of a
        head share every uniform (common random numbers).  Each row keeps its
        own inclusion probabilities, so its draw is marginally the same Poisson
        sample and its estimate stays unbiased; a block lands in both lists with
        probability min(pi_0, pi_1) instead of pi_0*pi_1, so the two rows, which
        abatt_attention processes together, gather more blocks once for both. */
enum { ABATT_DRAWS_INDEPENDENT = 0, ABATT_DRAWS_PAIRED = 1 };

/* Memory layout of Q, K, V and O.
   BHND: [B][H][N][d] -- each head's tokens contiguous.
   BNHD: [B][N][H][d] -- token-major with the heads interleaved, as the
        query/key/value projections of a transformer block emit them and its
        output projection reads them, so no transpose is needed around a call.
   Results are bit-identical between the two layouts. */
enum { ABATT_LAYOUT_BHND = 0, ABATT_LAYOUT_BNHD = 1 };

/* How abatt_select scores the key blocks for a query block's centroids c_j.
   KEYS: every key -- the block's share of centroid j's softmax over all keys.
   BLOCK_MEANS: the coarse-summary baseline the abstract contrasts with -- each
        block once, through the mean kbar_b of its keys, its share taken as
        n_b * exp(scale * c_j . kbar_b) normalised over the blocks (n_b = valid
        keys of b); Bk times less scoring work. */
enum { ABATT_SCORE_KEYS = 0, ABATT_SCORE_BLOCK_MEANS = 1 };

typedef struct abatt_config {
    int q_block;        /* Bq: queries per query block (128) */
    int kv_block;       /* Bk: keys per key/value block (16 by default) */
    int clusters;       /* C: k-means clusters per query block */
    int kmeans_iters;   /* I: Lloyd rounds (assign + update) */
    int budget_bp;      /* expected drawn blocks, basis points of nK:
                           M = floor((budget_bp*nK + 5000)/10000); M >= nK
                           keeps every block with weight 1 */
    float scale;        /* softmax scale s (1/sqrt(d) for plain attention) */
    uint64_t seed;      /* Philox key for the draws */
    int batch_offset;   /* global index of this call's first batch element (0 for a whole tensor) */
    int head_offset;    /* global index of this call's first head (0 for a whole tensor) */
    int selection;      /* ABATT_SELECT_SIP (0, the method) or ABATT_SELECT_TOPK (1) */
    int scoring;        /* ABATT_SCORE_KEYS (0, the method as read) or ABATT_SCORE_BLOCK_MEANS (1) */
    int layout;         /* ABATT_LAYOUT_BHND (0) or ABATT_LAYOUT_BNHD (1) */
    int draws;          /* ABATT_DRAWS_INDEPENDENT (0) or ABATT_DRAWS_PAIRED (1) */
    /* The sampler's Philox counter uses the global indices (beta + batch_offset,
       h + head_offset), so a call over a slice of the batches or heads of a
       larger problem draws exactly the blocks that one call over the whole
       problem draws for that slice.  Both must be >= 0 (ABATT_ERR_INVALID_ARG).
       selection, scoring, layout and draws outside their listed values also
       return ABATT_ERR_INVALID_ARG, before any launch. */
} abatt_config;

/* Which call a workspace is for. */
typedef enum abatt_call {
    ABATT_CALL_SELECT = 0,
    ABATT_CALL_SAMPLE = 1,
    ABATT_CALL_ATTENTION = 2,
    ABATT_CALL_FORWARD = 3
} abatt_call;

/* Bytes of device workspace `call` needs for this shape/config (256-byte
 * aligned base; it does not depend on the list capacity).  Host-only, no
 * CUDA call. */
abatt_status abatt_workspace_size(abatt_call call, const abatt_shape *shape,
                                  const abatt_config *cfg, size_t *bytes);

/* IBCS (abstract, selector sentence): for every query block, Lloyd k-means of
 * its valid queries (C_eff = min(C, n) clusters seeded at rows
 * floor(j*n/C_eff), ties to the lower index, empty clusters keep their
 * centroid), then each centroid's softmax (scale s) mass over all keys,
 * summed per key block and weighted by the cluster's share n_j/n:
 *   p[row][b] = sum_j (n_j/n) * sum_{t in block b} softmax_t(s c_j . k_t).
 * Output p: fp32 [B*H*nQ][nK], each row sums to 1.
 * Optional outputs (NULL to skip): centroids fp32 [B*H*nQ][C][d] and
 * cluster sizes int32 [B*H*nQ][C] (0 for unused clusters). */
abatt_status abatt_select(const void *Q, const void *K, const abatt_shape *shape,
                          const abatt_config *cfg, float *p, float *centroids,
                          int32_t *cluster_sizes, void *workspace, size_t workspace_bytes,
                          void *stream);

/* SIP (abstract, sampling sentence): Poisson draw of key blocks per row with
 * inclusion probabilities pi_b = min(1, c p_b), sum_b pi_b = M, solved
 * exactly in 48-bit fixed point (P_b = round-half-even(p_b 2^48), p clamped
 * to [0,1], NaN read as 0; water-filling of the saturated set).  Draw U_b is
 * word (b mod 4) of Philox4x32-10 at counter (b/4, i, h, beta) (i/2 in
 * place of i with ABATT_DRAWS_PAIRED), key
 * (seed lo, seed hi); block b is taken iff saturated or U_b/2^32 < pi_b
 * (exact integer test).
 * Outputs: counts int32 [rows]; idx int32 [rows][capacity] in ascending
 * order; logw fp32 [rows][capacity] = -ln(pi_b) (0 when pi_b = 1).  A row
 * that draws more than `capacity` blocks keeps the first `capacity` and sets
 * ABATT_DEVFLAG_CAPACITY.  Results are bit-identical for any launch
 * configuration, stream or device. */
abatt_status abatt_sample(const float *p, const abatt_shape *shape, const abatt_config *cfg,
                          int32_t *counts, int32_t *idx, float *logw, int capacity,
                          void *workspace, size_t workspace_bytes, void *stream);

/* Gather attention (abstract, kernel sentence): for every query block, exact
 * softmax attention over the keys of its listed blocks only, each logit of
 * block b shifted by logw_b:
 *   O[q] = sum_t e^{l_t} v_t / sum_t e^{l_t},  l_t = s q.k_t + logw_{b(t)}.
 * Each row's list must be strictly ascending (as abatt_sample writes it).
 * Blocks are gathered from K/V into 128-key tensor-core tiles.  Two
 * neighbouring query blocks (rows 2p, 2p+1 of a head) run together: their
 * lists are laid out as [blocks both drew | row 2p only | row 2p+1 only]; each
 * row walks exactly its own blocks ([both | its own]) in tiles of 128/kv_block
 * blocks, so no tile holds a block the row did not draw, and the tiles that
 * lie wholly inside the shared segment are gathered once for both rows.  An
 * empty list gives O = 0 (and lse = -inf).  lse (optional, NULL to skip):
 * fp32 [B][H][N], natural-log sum of exponentials per query.  Indices outside
 * [0, nK) or out of order are skipped and flagged ABATT_DEVFLAG_BADLIST.
 * This is abatt_attention_plan followed by abatt_attention_planned. */
abatt_status abatt_attention(const void *Q, const void *K, const void *V,
                             const abatt_shape *shape, const abatt_config *cfg,
                             const int32_t *counts, const int32_t *idx, const float *logw,
                             int capacity, void *O, float *lse, void *workspace,
                             size_t workspace_bytes, void *stream);

/* The two launches of abatt_attention, for callers that time or repeat them
 * separately.  abatt_attention_plan clears the workspace status word and
 * lays every pair's lists out in the ATTENTION workspace (segment lengths,
 * the pair's block array, each row's base-2 log-weights in its walking
 * order); abatt_attention_planned runs the gather-attention kernel from that
 * plan and does not clear the status word.  The plan stays valid while the
 * workspace is not reused by another call; Q, K, V may change between
 * planned calls.  Arguments as for abatt_attention. */
abatt_status abatt_attention_plan(const abatt_shape *shape, const abatt_config *cfg,
                                  const int32_t *counts, const int32_t *idx, const float *logw,
                                  int capacity, void *workspace, size_t workspace_bytes,
                                  void *stream);
abatt_status abatt_attention_planned(const void *Q, const void *K, const void *V,
                                     const abatt_shape *shape, const abatt_config *cfg, void *O,
                                     float *lse, void *workspace, size_t workspace_bytes,
                                     void *stream);

/* The whole path: select -> sample -> attention, on one stream, with p and the
 * lists kept in the workspace (capacity nK, so no row can overflow). */
abatt_status abatt_forward(const void *Q, const void *K, const void *V,
                           const abatt_shape *shape, const abatt_config *cfg, void *O,
                           float *lse, void *workspace, size_t workspace_bytes, void *stream);

/* Pointers into a FORWARD workspace (valid after abatt_forward completes):
 * p fp32 [rows][nK], counts int32 [rows], idx int32 [rows][nK],
 * logw fp32 [rows][nK].  Any output pointer may be NULL. */
abatt_status abatt_forward_intermediates(void *workspace, const abatt_shape *shape,
                                         const abatt_config *cfg, float **p, int32_t **counts,
                                         int32_t **idx, float **logw);

/* Gather attention without a workspace, for callers that cannot allocate
 * device memory: for example code running inside a memory pool or arena it
 * does not own, a plugin whose host application forbids allocation during
 * inference, or a process that must not trigger allocation (and its
 * synchronisation) on a latency-critical path.  No counterpart in the paper:
 * this is an interface convenience of this library.
 *
 * Computes exactly what abatt_attention computes, with the same arguments
 * except the workspace.  Its scratch (status word and the per-pair union
 * lists) lives in a fixed array of ABATT_NOALLOC_SCRATCH_BYTES inside the
 * library's device image; every GPU that loads the library holds that
 * array until the process exits.  Shapes whose scratch would exceed it are
 * rejected with ABATT_ERR_UNSUPPORTED before any launch (the scratch needed
 * is abatt_workspace_size(ABATT_CALL_ATTENTION, ...)).
 *
 * The array's device address is looked up with cudaGetSymbolAddress the
 * first time the call runs in a CUDA context (the current device's), and
 * cached for that context only: a call from another context (after
 * cudaDeviceReset, or one a host created with the driver API) looks it up
 * again.  Make the first call in each context before any stream capture.
 * Every call on a device shares the one array and leaves its contents
 * behind: calls that may overlap on the GPU (different streams without
 * ordering, or concurrent host threads) race on it and must be serialised by
 * the caller.  The call allocates and frees nothing.
 *
 * dev_status (device pointer, NULL to skip): once the arguments pass the
 * host checks, it is set to ABATT_NOALLOC_STATUS_PENDING (all bits) on
 * `stream`, and replaced by the ABATT_DEVFLAG_* bits of this call when every
 * launch of the call was enqueued; if the call returns an error after that
 * point, it keeps the PENDING value. */
#define ABATT_NOALLOC_STATUS_PENDING 0xFFFFFFFFu
#define ABATT_NOALLOC_SCRATCH_BYTES (64u << 20)
abatt_status abatt_attention_noalloc(const void *Q, const void *K, const void *V,
                                     const abatt_shape *shape, const abatt_config *cfg,
                                     const int32_t *counts, const int32_t *idx, const float *logw,
                                     int capacity, void *O, float *lse, uint32_t *dev_status,
                                     void *stream);

/* Test hooks (no counterpart in the paper).  They let the tests drive the
 * failure path of the bounded device waits without faulting a GPU, and check
 * the FMA-pipe exponential the kernels use, against CUDA's exp2f.
 *   abatt_test_set(ABATT_TEST_WAIT_NS, ns): limit of every bounded wait of
 *        later calls, in nanoseconds (0 restores the default, 0.5 s).
 *   abatt_test_set(ABATT_TEST_STALL, mask): the copy producer of the
 *        attention kernel (bit ABATT_TEST_STALL_ATTENTION) or of the scoring
 *        kernel (ABATT_TEST_STALL_SCORE) stops after its first tile, so the
 *        waits for later tiles run out: the call sets ABATT_DEVFLAG_TIMEOUT,
 *        its CTAs drain what they issued, free tensor memory and return.  0
 *        turns it off.
 * Process-wide; not safe against calls running concurrently on other host
 * threads.  ABATT_ERR_INVALID_ARG for an unknown hook. */
enum { ABATT_TEST_WAIT_NS = 1, ABATT_TEST_STALL = 2 };
#define ABATT_TEST_STALL_ATTENTION 0x1u
#define ABATT_TEST_STALL_SCORE 0x2u
abatt_status abatt_test_set(int hook, uint64_t value);

/* y[i] = 2^x[i] through the kernels' FMA-pipe polynomial of the given degree
 * (3 or 4): Cody-Waite reduction x = j + f and a minimax polynomial for 2^f
 * with constant term 1; inputs at or below -127 give +0.  x and y are device
 * fp32 arrays of n elements; asynchronous on `stream`. */
abatt_status abatt_test_exp2_poly(const float *x, float *y, int64_t n, int degree, void *stream);

/* Synchronously copy the device status word at the start of `workspace` to
 * *flags (ABATT_DEVFLAG_* bits) after `stream` drains.  Returns
 * ABATT_ERR_DEVICE if any bit is set, ABATT_OK otherwise. */
abatt_status abatt_read_status(const void *workspace, uint32_t *flags, void *stream);

/* Zero the device status word (asynchronous on `stream`). */
abatt_status abatt_clear_status(void *workspace, void *stream);

/* Static description of a status code. */
const char *abatt_status_string(abatt_status s);

/* Library version "major.minor.patch". */
const char *abatt_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ABATT_H */
