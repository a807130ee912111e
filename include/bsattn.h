/*
 * libbsattn — block-sparse (keep-or-drop) and piecewise (PISA) attention for
 * diffusion transformers on one NVIDIA B200 (sm_100a).
 *
 * Sources (page title and section):
 *   [BSA]  "多模态 DiT 上的块稀疏 Attention" (block-sparse attention on multimodal DiT,
 *          dpshk.com engineering blog): §3.3 block-sparse output formula, §4.1 block
 *          layout (text first, image after, each padded to a block multiple), §4.2 the
 *          multimodal fixed pattern, §4.3/§4.4 the per-query-block loop with online
 *          softmax, §5.4 index lists instead of a dense mask, §8.1 build once / reuse.
 *   [PISA] "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
 *          Transformers" (gist.science summary of arXiv 2602.01077), technical summary
 *          §2: exact-or-approximate split S_i / U_i, o_t = N_t / D_t, zeroth-order
 *          centroid terms alpha_{t,j}, global first-order correction with H-bar,
 *          covariance-aware routing with M_j = ||H_j - H-bar||, and the fused pipeline
 *          (precompute -> exact stage -> zeroth-order sweep -> first-order correction).
 *
 * Conventions shared by every call
 *   - Tensors are contiguous, row-major [Bt, H, L, d] (page [BSA] §4.3 uses
 *     q, k, v: [B, H, N, D]); Q, K, V and O are bf16; statistics are fp32.
 *     "BH" below is Bt * H, "M" is L / block.
 *   - Every pointer except `desc` is a DEVICE pointer the caller allocated; the
 *     library never allocates, frees or synchronises. Device buffers must be 16-byte
 *     aligned.
 *   - Every call is asynchronous on `stream` (a cudaStream_t, NULL = legacy default
 *     stream). The return value reports host-side argument validation and launch
 *     errors only.
 *   - `status` (nullable) is one device int32 the caller zeroes. Kernels that detect
 *     a data error (malformed block lists, overflowing capacity, a wait that timed
 *     out) write the first such bsa_status code there and never trap. A call whose
 *     inputs were found malformed leaves its outputs unwritten.
 *   - Supported: d in {64, 128}; block in {64, 128}; L % block == 0; M <= 2048.
 *     Anything else returns BSA_ERR_UNSUPPORTED.
 *   - Token padding ([BSA] §4.1 pads the text segment to a multiple of the block size;
 *     §7.3 gives a timestep token its own block): `key_valid` (nullable, device int32
 *     [M], shared by every (batch, head)) is the number of leading real tokens of each
 *     block, 1..block; the rest of the block is padding. NULL means no padding. Padded
 *     keys receive no attention weight; centroids, value sums, H_j and pooled queries
 *     are taken over real tokens only; an unselected block's Taylor-tail weight is its
 *     real-token count; a padded block is always computed exactly: bsa_route places it
 *     in every list, and bsa_forward in the PISA modes reports BSA_ERR_BAD_PADDING for a
 *     list that lacks one. Padded query rows are computed like any other row. Values
 *     outside 1..block report BSA_ERR_BAD_PADDING (and are clamped). A key_valid
 *     pointer that is not 4-byte aligned returns BSA_ERR_INVALID_ARG.
 */
#ifndef BSATTN_H
#define BSATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BSA_API __attribute__((visibility("default")))
#else
#define BSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, non-positive size, ...     */
  BSA_ERR_UNSUPPORTED = 2,   /* valid request outside the supported shapes          */
  BSA_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed          */
  BSA_ERR_BAD_CSR = 4,       /* block lists malformed (device-detected)              */
  BSA_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up (device-detected) */
  BSA_ERR_WORKSPACE = 6,     /* workspace null or smaller than bsa_workspace_bytes   */
  BSA_ERR_CAPACITY = 7,      /* an output list would exceed its capacity (device)    */
  BSA_ERR_SCRATCH_LIMIT = 8, /* bsa_forward_noalloc: the shape needs more scratch than
                                BSA_NOALLOC_SCRATCH_BYTES                            */
  BSA_ERR_BAD_PADDING = 9    /* key_valid out of range, or a padded block missing from a
                                PISA list (device-detected)                          */
} bsa_status;

/* Size of the device scratch array built into the library for bsa_forward_noalloc. */
#define BSA_NOALLOC_SCRATCH_BYTES (16u << 20)

typedef enum {
  BSA_MODE_KEEP_OR_DROP = 0, /* [BSA] §3.3: softmax over the selected blocks only      */
  BSA_MODE_PISA = 1,         /* [PISA] §2: exact S_i + Taylor-approximated U_i         */
  BSA_MODE_PISA_BLOCK = 2    /* [PISA] §2, first order with each block's own H_j       */
} bsa_mode;

typedef enum {
  BSA_CALL_BUILD_MASK = 0,
  BSA_CALL_PRECOMPUTE = 1,
  BSA_CALL_ROUTE = 2,
  BSA_CALL_FORWARD = 3
} bsa_call;

/* Multimodal fixed pattern, [BSA] §4.2, generalised from the page's 1-D image
 * sequence to a 2-D grid of image blocks.
 *   n_text_blocks    text blocks at the front of the sequence ([BSA] §4.1 puts text
 *                    first, each modality padded to a block multiple);
 *   grid_h, grid_w   image blocks form a grid_h x grid_w grid, row-major;
 *   radius           image block a keeps image block b when the Chebyshev distance
 *                    of their grid positions is <= radius (radius 1 = 3x3 window;
 *                    grid_h 1 reproduces the page's |i - j| <= window_size);
 *   global_stride    image block b is global (kept by every image row) when
 *                    b % global_stride == 0; 0 disables global blocks;
 *   global_rows_full nonzero: global image blocks also keep every block.
 * Text rows and text columns are always full. M = n_text_blocks + grid_h*grid_w. */
typedef struct {
  int32_t n_text_blocks;
  int32_t grid_h;
  int32_t grid_w;
  int32_t radius;
  int32_t global_stride;
  int32_t global_rows_full;
} bsa_mask_desc;

/* Library version (major * 10000 + minor * 100 + patch). */
BSA_API int32_t bsa_version(void);

/* Human-readable name of a bsa_status code (static string, never NULL). */
BSA_API const char* bsa_status_string(int32_t code);

/* Number of blocks M of a mask descriptor, or -1 if the descriptor is invalid. */
BSA_API int32_t bsa_mask_blocks(const bsa_mask_desc* desc);

/* Bytes of device workspace a call needs for the given shape (0 = none). `call` is
 * a bsa_call; the sizes are those of the corresponding call. Returns 0 for an
 * unsupported shape. */
BSA_API size_t bsa_workspace_bytes(int32_t call, int32_t Bt, int32_t H, int32_t L, int32_t d,
                           int32_t block);

/* bsa_build_mask — the multimodal fixed pattern as CSR block lists ([BSA] §4.2,
 * stored as index lists per [BSA] §5.4; built once and reused per [BSA] §8.1).
 *   desc      host pointer to the pattern descriptor;
 *   row_ptr   device int32[M + 1]: row i's key blocks are col_idx[row_ptr[i] ..
 *             row_ptr[i+1]); row_ptr[0] = 0;
 *   col_idx   device int32[col_capacity], written strictly ascending per row;
 *             M*M always suffices;
 *   status    see conventions; BSA_ERR_CAPACITY if nnz > col_capacity (then only
 *             row_ptr is written).
 * One shared list serves every (batch, head) ([BSA] §8.2). */
BSA_API bsa_status bsa_build_mask(const bsa_mask_desc* desc, int32_t* row_ptr, int32_t* col_idx,
                          int64_t col_capacity, int32_t* status, void* stream);

/* bsa_precompute — per-block statistics of [PISA] §2 ("precompute" stage):
 *   kbar_j = (1/B_j) sum_n k_{j,n}                   -> kbar  fp32 [BH, M, d]
 *   vsum_j = sum_n v_{j,n}                           -> vsum  fp32 [BH, M, d]
 *   H_j    = sum_n (k_{j,n} - kbar_j)^T v_{j,n}      (d_k rows x d_v cols)
 *   Hbar   = (1/M) sum_j H_j  (mean over all blocks of the head) -> Hbar fp32 [BH, d, d]
 *   Mnorm_j = ||H_j - Hbar||_F (Frobenius)           -> Mnorm fp32 [BH, M]
 *   Hblk (nullable) receives every H_j              -> fp32 [BH, M, d, d]
 *   (sums over the B_j real tokens of block j: B_j = key_valid[j], or B)
 * K, V are bf16 [Bt, H, L, d]. workspace: device, >= bsa_workspace_bytes(
 * BSA_CALL_PRECOMPUTE, ...) bytes, contents scratch. */
BSA_API bsa_status bsa_precompute(const void* K, const void* V, int32_t Bt, int32_t H, int32_t L,
                          int32_t d, int32_t block, const int32_t* key_valid, float* kbar,
                          float* vsum, float* Hbar, float* Mnorm, float* Hblk,
                          void* workspace, size_t ws_bytes, int32_t* status, void* stream);

/* bsa_route — covariance-aware top-k block selection ([PISA] §2, routing).
 *   qbar_i   = mean of the (real) queries of block i;
 *   p_ij     = softmax_j(scale * qbar_i . kbar_j) over all M key blocks;
 *   score_ij = p_ij + lambda * Mnorm_j / sum_j' Mnorm_j'  (term is 0 if the sum is 0);
 *   S_i      = the padded blocks, then the highest scores up to k_top, ties to the
 *              smaller j, written ascending (BSA_ERR_BAD_PADDING if k_top is smaller
 *              than the number of padded blocks).
 * (The pages say the score "combines" the attention score with M_j without a
 * formula; this mix of two distributions is this library's reading.)
 *   Q        bf16 [Bt, H, L, d];  kbar fp32 [BH, M, d];  Mnorm fp32 [BH, M];
 *   scale    score scale; 0 selects 1/sqrt(d);
 *   row_ptr  device int32 [BH, M + 1]: absolute offsets into col_idx; head h row i is
 *            col_idx[row_ptr[h*(M+1)+i] .. row_ptr[h*(M+1)+i+1]) = h*M*k_top + i*k_top ..;
 *   col_idx  device int32 [BH, M * k_top];
 *   scores   nullable fp32 [BH, M, M] receives score_ij;
 *   workspace  device, >= bsa_workspace_bytes(BSA_CALL_ROUTE, ...) bytes (the column sums
 *            of every 32-row segment of Q, BH * L/32 * d floats), contents scratch.
 * 1 <= k_top <= M. */
BSA_API bsa_status bsa_route(const void* Q, const float* kbar, const float* Mnorm, int32_t Bt,
                     int32_t H, int32_t L, int32_t d, int32_t block, const int32_t* key_valid,
                     int32_t k_top, float lambda, float scale, int32_t* row_ptr,
                     int32_t* col_idx, float* scores, void* workspace, size_t ws_bytes,
                     int32_t* status, void* stream);

/* bsa_forward — fused online-softmax attention over block lists.
 *   mode BSA_MODE_KEEP_OR_DROP ([BSA] §3.3):
 *     o_t = sum_{j in S_i} sum_n e^{s q.k_{j,n}} v_{j,n} / sum_{j in S_i} sum_n e^{s q.k_{j,n}}
 *     A row with an empty list outputs zeros and lse = -inf.
 *   mode BSA_MODE_PISA ([PISA] §2), with alpha_tj = e^{s q_t.kbar_j}:
 *     N_t = sum_{S_i} sum_n e^{s q.k} v + sum_{U_i} alpha_tj vsum_j
 *           + s (q_t Hbar) sum_{U_i} alpha_tj
 *     D_t = sum_{S_i} sum_n e^{s q.k} + sum_{U_i} block * alpha_tj;   o_t = N_t / D_t
 *     (every exponent is shifted by a running row maximum, which cancels).
 *   mode BSA_MODE_PISA_BLOCK ([PISA] §2, the per-block first-order term, of which the
 *     Hbar form above is the global approximation):
 *     N_t = sum_{S_i} sum_n e^{s q.k} v + sum_{U_i} alpha_tj (vsum_j + s q_t H_j)
 *     D_t as for BSA_MODE_PISA. Because kbar_j is the mean key of block j, s q_t.kbar_j
 *     is the mean of the row's exact scores over the block, and
 *     alpha_tj (vsum_j + s q_t H_j) = sum_n alpha_tj (1 + s q_t.(k_{j,n} - kbar_j)) v_{j,n}:
 *     every unselected block is computed as a tile whose weights are the first-order
 *     expansion of e^{s q.k} about its centroid. No statistics are read (kbar, vsum,
 *     Hbar may be NULL); every block of every query block is a tile, so the tensor
 *     work is that of dense attention: an accuracy reference, not a fast path.
 *   Q, K, V      bf16 [Bt, H, L, d];   O bf16 [Bt, H, L, d] (written);
 *   row_ptr/col_idx  block lists, each row strictly ascending in [0, M);
 *     csr_per_head 0: one list of M rows (row_ptr int32[M+1]) shared by every head;
 *     csr_per_head 1: per-head lists laid out as bsa_route writes them;
 *   nnz_total    number of entries in col_idx (bounds every row_ptr value);
 *   kbar, vsum, Hbar  bsa_precompute outputs (PISA only; ignored, may be NULL, for
 *                keep-or-drop);
 *   scale        0 selects 1/sqrt(d);
 *   lse          nullable fp32 [BH, L]: natural-log denominator, m_t + log D_t;
 *   workspace    device, >= bsa_workspace_bytes(BSA_CALL_FORWARD, ...) bytes.
 *   key_valid    see the conventions: padded keys are masked; in the PISA modes every
 *                padded block must be in every list.
 * Malformed lists set BSA_ERR_BAD_CSR (a missing padded block BSA_ERR_BAD_PADDING) in
 * *status and leave O unwritten. */
BSA_API bsa_status bsa_forward(const void* Q, const void* K, const void* V, int32_t Bt, int32_t H,
                       int32_t L, int32_t d, int32_t block, const int32_t* key_valid,
                       const int32_t* row_ptr,
                       const int32_t* col_idx, int64_t nnz_total, int32_t csr_per_head,
                       int32_t mode, const float* kbar, const float* vsum,
                       const float* Hbar, float scale, void* O, float* lse,
                       void* workspace, size_t ws_bytes, int32_t* status, void* stream);

/* bsa_forward_noalloc — bsa_forward for callers that cannot allocate device memory.
 * (No counterpart in the pages: this is a deployment variant of bsa_forward.)
 * Some callers cannot call cudaMalloc: a host whose memory pool owns the whole device
 * and forbids allocations from plug-ins, a serving loop that cannot take cudaMalloc's
 * implicit synchronisation, an embedded runtime with a memory budget fixed at load time.
 * This call takes the same arguments as bsa_forward minus the workspace and computes
 * the same result; its scratch is one __device__ array of BSA_NOALLOC_SCRATCH_BYTES
 * inside the library, which every GPU that loads the library keeps until the process
 * exits. It calls no allocating routine.
 *   - The scratch address is looked up on the current device at every call (the device
 *     of the stream); the first call on a device may load the library's device code, so
 *     make it before any stream capture.
 *   - Every call shares the one array (per device) and leaves its contents behind; calls
 *     whose kernels overlap on the GPU (different streams or host threads) race on it,
 *     so serialise them.
 *   - Returns BSA_ERR_SCRATCH_LIMIT when the shape needs more scratch than the array
 *     holds: PISA needs 256 + 2*BH*Mp*d*2 + BH*d*d*2 bytes (Mp = M rounded up to 128,
 *     each term rounded up to 256), the other modes 256 bytes. Other errors as bsa_forward. */
BSA_API bsa_status bsa_forward_noalloc(const void* Q, const void* K, const void* V, int32_t Bt,
                                       int32_t H, int32_t L, int32_t d, int32_t block,
                                       const int32_t* key_valid, const int32_t* row_ptr,
                                       const int32_t* col_idx,
                                       int64_t nnz_total, int32_t csr_per_head, int32_t mode,
                                       const float* kbar, const float* vsum, const float* Hbar,
                                       float scale, void* O, float* lse, int32_t* status,
                                       void* stream);

/* bsa_selftest_wait_timeout — the failure path of every kernel, exercised without a fault.
 * (No counterpart in the pages.) Every wait of the library's kernels is bounded: a wait
 * that runs out sets a CTA-wide abort flag, the kernel drains and returns, and
 * BSA_ERR_TIMEOUT is written to *status, leaving the context usable. This call launches
 * one CTA whose thread waits, with that same bounded wait and a limit of timeout_ns, on
 * an mbarrier that nothing ever completes; the wait runs out and the kernel reports.
 *   timeout_ns  1 .. 10^10 (10 s); status: device int32, written with BSA_ERR_TIMEOUT.
 * Returns BSA_ERR_INVALID_ARG for a null status or a limit out of range. */
BSA_API bsa_status bsa_selftest_wait_timeout(int64_t timeout_ns, int32_t* status, void* stream);

/* bsa_selftest_forward_timeout — the attention kernel's own abort path, run without a fault.
 * (No counterpart in the pages.) The same launch sequence as bsa_forward (per-head lists,
 * no token padding, default scale, no lse), with every bounded wait of the attention
 * kernel limited to wait_ns instead of its 2 s default. With a limit far below the time
 * the kernel's copies and MMAs take, a wait runs out while TMA copies and tensor-core work
 * are in flight: the CTA raises its abort flag, every role leaves its loop, the producer
 * drains its copies, the MMA thread waits for its issued MMAs, TMEM is freed and
 * BSA_ERR_TIMEOUT is written to *status. O is then partly written (unspecified); the
 * context stays usable.
 *   wait_ns  1 .. 10^10; status: device int32 the caller zeroes (required); other
 *            arguments as bsa_forward. */
BSA_API bsa_status bsa_selftest_forward_timeout(const void* Q, const void* K, const void* V,
                                                int32_t Bt, int32_t H, int32_t L, int32_t d,
                                                int32_t block, const int32_t* row_ptr,
                                                const int32_t* col_idx, int64_t nnz_total,
                                                int32_t mode, const float* kbar,
                                                const float* vsum, const float* Hbar, void* O,
                                                void* workspace, size_t ws_bytes,
                                                int64_t wait_ns, int32_t* status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BSATTN_H */
