/*
 * sparse_attn — block-sparse attention, forward and backward, for NVIDIA B200 (sm_100a).
 *
 * C ABI.  Plain pointers and sizes only; no C++ or framework types cross it.
 * Every call returns an int status (SA_OK or a negative SA_ERR_* code); no
 * exception or abort crosses the boundary.  The caller owns every buffer.
 *
 * The computation.  Scaled dot-product attention in which query q may attend
 * only to keys kv allowed by a fixed pattern, with the softmax taken over the
 * allowed keys alone.  The pattern and the masked-softmax definition follow:
 *   - "Sparse Attention" glossary page (ultralytics.com/de/glossary/sparse-attention),
 *     section "Gängige Sparsity-Muster": sliding window, every s-th prior token,
 *     global tokens, attention sinks;
 *   - the same page, section "Ein Muster in Einsparungen verwandeln": the
 *     local_plus_sinks predicate (causal, q - kv <= window, or kv < sinks), its
 *     compilation into 128 x 128 blocks, and kernels that skip the empty ones;
 *   - "Sparse-трансформеры: как урезать O(n²) внимания" (1gpt.online), section
 *     "Как это выглядит в коде": scores q.k / sqrt(d), -inf outside the mask,
 *     softmax, times V.
 *
 * Tensor layouts (all contiguous, row-major):
 *   Q, O  [B, Hq,  N, D] bf16        K, V  [B, Hkv, N, D] bf16
 *   LSE   [B, Hq,  N]    fp32        natural log of the softmax denominator,
 *                                    sum over allowed kv of exp(scale * q.k)
 * Query head hq reads key/value head hq / (Hq / Hkv).
 */
#ifndef SPARSE_ATTN_H
#define SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
#define SA_OK 0
#define SA_ERR_INVALID_ARG (-1)      /* null pointer, negative size, bad scale */
#define SA_ERR_UNSUPPORTED (-2)      /* D not in {64, 128}, block not in {64, 128}, Hq % Hkv != 0, a pattern form not built */
#define SA_ERR_MISALIGNED (-3)       /* a tensor pointer is not 16-byte aligned */
#define SA_ERR_BUFFER_TOO_SMALL (-4) /* output arrays smaller than the tile count */
#define SA_ERR_CUDA (-5)             /* a CUDA runtime call or kernel launch failed */
#define SA_ERR_DEVICE_TIMEOUT (-6)   /* a bounded wait inside the kernel expired */
#define SA_ERR_MASK_MISMATCH (-7)    /* block mask built for another N or block */
#define SA_ERR_SCRATCH_TOO_SMALL (-8) /* sparse_attn_fwd_noalloc: mask larger than its static scratch */

/*
 * A fixed sparsity pattern.  A pair (q, kv) is allowed when
 *     (causal == 0 or q >= kv)
 *     and ( (window >= 0 and |q - kv| <= window)
 *           or kv < sinks
 *           or (stride > 0 and (q - kv) mod stride == 0)
 *           or kv < n_global or q < n_global
 *           or (area > 0 and floor(q / area) == floor(kv / area))
           or (area > 0 and summary > 0 and kv mod area >= area - summary) ).
 * Pages: "Sparse Attention", sections "Gängige Sparsity-Muster" and "Ein
 * Muster in Einsparungen verwandeln" (window inclusive, as in local_plus_sinks),
 * and section "Anwendungen" (Area Attention: attention only inside stripes of
 * consecutive tokens); "Sparse-трансформеры", section "Основные шаблоны
 * разреженности" (without causality the window reaches w tokens on both
 * sides), and the "fixed" pattern of the same section: blocks of `area`
 * tokens with local attention inside, linked through summary positions, read
 * as the last `summary` positions of every block.  The stride counts back from
 * the query (every s-th prior token) and
 * needs causal == 1; with causal == 1 the global rows and columns stay causal.
 * Supported forms: causal == 1 with any of the rules; causal == 0 with window,
 * sinks, n_global, area and summary (stride > 0 gives SA_ERR_UNSUPPORTED, as
 * does a stride with area); summary > 0 needs area > 0 (SA_ERR_INVALID_ARG).
 */
typedef struct {
    int32_t causal;
    int32_t window;
    int32_t sinks;
    int32_t stride;
    int32_t n_global;
    int32_t area;     /* stripe (block) length; 0 for none */
    int32_t summary;  /* summary positions at the end of every stripe; 0 for none */
} sa_pattern;

/*
 * The compiled pattern: for every query tile i (block rows) the ascending list
 * of kv tiles that hold at least one allowed pair, and for each a flag that is
 * 1 when every in-range pair of the tile is allowed (the kernel then skips the
 * per-element mask).  Arrays are row-major with row stride n_kv_tiles:
 *   kv_count[i]                number of listed tiles of row i
 *   kv_index[i*n_kv_tiles + c] c-th listed kv tile, ascending; -1 after the last
 *   kv_full [i*n_kv_tiles + c] 1 full, 0 partial; 0 after the last
 * The last tile of each side is ragged when block does not divide N; only its
 * in-range pairs count.  Pages: "Sparse Attention", section "Ein Muster in
 * Einsparungen verwandeln" (create_block_mask and its 128 x 128 blocks).
 */
typedef struct {
    int32_t n_q_tiles;   /* builder: in = capacity of rows, out = T */
    int32_t n_kv_tiles;  /* builder: in = capacity of a row, out = T (the row stride) */
    int32_t block;       /* out: tile edge */
    int32_t max_per_row; /* out: largest kv_count */
    int64_t n_live;      /* out: sum of kv_count */
    int64_t n_full;      /* out: number of full tiles */
    int32_t* kv_count;
    int32_t* kv_index;
    uint8_t* kv_full;
} sa_block_mask;

typedef struct {
    int32_t B, Hq, Hkv, N, D;
} sa_shape;

/* T = ceil(N / block), the number of tiles per side; negative status on a bad argument. */
int32_t sparse_attn_num_tiles(int64_t N, int32_t block);

/*
 * Classify every (q-tile, kv-tile) pair of an N x N score matrix as empty,
 * partial or full and write the lists described at sa_block_mask: for causal
 * patterns without stripes analytically per tile (no per-pair or per-row
 * loop); for the others (causal == 0, or area > 0) from each row's allowed
 * keys, a union of at most four intervals plus the periodic summary columns,
 * counted per tile in closed form.  Host-only; `out` holds
 * caller-owned host arrays with capacity out->n_q_tiles rows of
 * out->n_kv_tiles entries, both at least T (else SA_ERR_BUFFER_TOO_SMALL).
 * block is 64 or 128; N >= 0 (N = 0 gives T = 0).
 */
int sparse_attn_build_block_mask(const sa_pattern* pattern, int64_t N, int32_t block, sa_block_mask* out);

/*
 * Number of allowed (q, kv) pairs of one head, 0 <= q, kv < N, in closed form
 * per query row (interval unions for the forms without a stride).  4 * D *
 * pairs is the useful work of one (batch, head).
 */
int sparse_attn_count_pairs(const sa_pattern* pattern, int64_t N, int64_t* pairs);

/*
 * Forward pass on the GPU.  Q, K, V, O, LSE are device pointers (Q, K, V, O
 * 16-byte aligned, LSE 4-byte aligned) in the layouts above; `mask` holds DEVICE copies of the arrays
 * built by sparse_attn_build_block_mask for this pattern, N and block (its
 * scalar fields as the builder returned them); arrays that the current device
 * cannot read (pageable host memory, another device's memory) are refused with
 * SA_ERR_INVALID_ARG before any launch.  scale > 0 multiplies q.k
 * (1/sqrt(D) in the pages' prototype).  `stream` is a cudaStream_t (NULL: the
 * legacy default stream).  Asynchronous: returns once the kernel is queued;
 * launch errors come back as SA_ERR_CUDA, a device-side timeout through
 * sparse_attn_check_device.  Rows with no allowed key get O = 0, LSE = -inf.
 * The first call on a device (of this or any other entry point that reports
 * through the status word) allocates the 4-byte device status word with
 * cudaMalloc and clears it, waiting for the device: that one call blocks the
 * host; later calls do not.  The kernels clamp a row's count to T and never
 * address a tile outside [0, T), whatever the device mask holds: a malformed
 * mask gives wrong results, not out-of-range accesses.  Results of the same
 * call on the same inputs are bit-identical.
 * Supported: D in {64, 128}, mask block in {64, 128}, Hq % Hkv == 0, the
 * pattern forms listed at sa_pattern, at most 4096 tiles per side (N <= 4096 *
 * block); else SA_ERR_UNSUPPORTED.  Patterns with causal == 0 or area > 0 run
 * on the kernel instantiation that takes a pattern table (as
 * sparse_attn_fwd_heads), which limits them to Hq <= 256.
 */
int sparse_attn_fwd(const void* Q, const void* K, const void* V, const sa_block_mask* mask,
                    const sa_pattern* pattern, const sa_shape* shape, float scale, void* O, float* LSE,
                    void* stream);

/*
 * The same forward pass from HOST buffers: Q, K, V, O, LSE and the block mask
 * (`mask_host`, the arrays as sparse_attn_build_block_mask returned them) are
 * all in host memory.  The mask is checked on the host first (counts in
 * [0, T], listed tiles strictly ascending in [0, T), flags 0 or 1; else
 * SA_ERR_INVALID_ARG, before any device work) and copied into `workspace`
 * (device memory, at least sparse_attn_fwd_host_workspace bytes, 256-byte
 * aligned).  The work is cut into chunks of whole key/value heads (with their
 * query heads), each half of the heads still left (the last takes one, at
 * most 16 chunks); chunk c + 1's inputs are copied in while chunk c computes
 * and chunk c - 1's O and LSE are copied back, on streams the library creates
 * once per device, ordered after the work already queued on `stream`.
 * Returns when everything is back in host memory (`stream` then waits on it
 * too), with the first error, including a device timeout.  Pinned host memory
 * makes the copies asynchronous DMA; pageable memory works but serialises
 * them.  Each chunk is a sparse_attn_fwd call on its heads: results are those
 * of sparse_attn_fwd, bit-identical when both calls split work units alike
 * (the kernel splits every unit of a problem with at most half as many units
 * as SMs, and those of a last round that would leave most CTAs idle).
 * Calls on one device are serialised.
 */
int sparse_attn_fwd_host(const void* Q_host, const void* K_host, const void* V_host, const sa_block_mask* mask_host,
                         const sa_pattern* pattern, const sa_shape* shape, float scale, void* O_host,
                         float* LSE_host, void* workspace, size_t workspace_bytes, void* stream);

/*
 * sparse_attn_fwd_host without the final wait: queues the same chunked copies
 * and kernels and returns; `stream` reaches the call's end once O and LSE are
 * in host memory.  Until then the caller must leave the host inputs, the host
 * mask and the workspace unchanged and must not read O_host, LSE_host.  Calls
 * on one device are ordered: a call's input copies wait only for the previous
 * call's kernels (not for its copies back), and its kernels for the previous
 * call's copies back, so successive steps overlap their input and output
 * copies.  Errors in the arguments come back at once; a device timeout through
 * sparse_attn_check_device.
 */
int sparse_attn_fwd_host_async(const void* Q_host, const void* K_host, const void* V_host,
                               const sa_block_mask* mask_host, const sa_pattern* pattern, const sa_shape* shape,
                               float scale, void* O_host, float* LSE_host, void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * Forward pass with a pattern per query head ("Sparse-трансформеры" page,
 * section "Комбинация — норма, а не исключение": heads of one layer may carry
 * different patterns, some local, some strided).  Query head h attends under
 * patterns[head_pattern[h]], with the block mask masks[head_pattern[h]]
 * compiled for it by sparse_attn_build_block_mask; a head's result is that of
 * sparse_attn_fwd under its own pattern.
 *
 *   masks        [n_patterns] block masks in DEVICE memory, all for the same N
 *                and block
 *   patterns     [n_patterns] (host), each as for sparse_attn_fwd
 *   n_patterns   1 .. 8
 *   head_pattern [Hq] (host) pattern index of each query head; Hq <= 256
 *   other arguments and layouts as sparse_attn_fwd; asynchronous on `stream`.
 *
 * Errors: SA_ERR_INVALID_ARG for a null argument, n_patterns out of range or
 * an index outside [0, n_patterns); SA_ERR_MASK_MISMATCH when the masks differ
 * in block or do not match N; SA_ERR_UNSUPPORTED for Hq > 256 and everything
 * sparse_attn_fwd rejects.
 */
int sparse_attn_fwd_heads(const void* Q, const void* K, const void* V, const sa_block_mask* masks,
                          const sa_pattern* patterns, int32_t n_patterns, const int32_t* head_pattern,
                          const sa_shape* shape, float scale, void* O, float* LSE, void* stream);

/* Device bytes sparse_attn_fwd_host needs for `shape`: Q, K, V, O, LSE and a
 * copy of a block mask of ceil(N / 64) tiles per side, each rounded up to 256
 * bytes. */
int sparse_attn_fwd_host_workspace(const sa_shape* shape, size_t* bytes);

/*
 * Wait for `stream`, then read and clear this device's kernel status word:
 * SA_ERR_DEVICE_TIMEOUT if a bounded wait inside a forward kernel gave up
 * since the last check, else SA_OK (or SA_ERR_CUDA if the wait failed).
 */
int sparse_attn_check_device(void* stream);

/*
 * Test hook.  flags: bit 0 makes the next forward launches (of every forward
 * entry point) skip the Q tile load, so the kernel's bounded waits expire and
 * it reports SA_ERR_DEVICE_TIMEOUT instead of computing.  Bit 1 makes sparse_attn_fwd
 * split every work unit (each query tile's kv list walked in two halves that
 * are merged at the end), the path the kernel otherwise takes only for small
 * problems and the last, partial round of units; results agree within
 * rounding.  Bit 2 makes
 * sparse_attn_bwd split every kv tile's list of more than 32 steps into work
 * items of at most 32 steps whose dK, dV add up in fp32 sums, the path it
 * otherwise takes only for lists longer than an SM's share of all steps.
 * timeout_cycles bounds every wait in SM clock cycles (<= 0 restores the
 * default, about one second).
 */
int sparse_attn_set_debug(int32_t flags, int64_t timeout_cycles);

/*
 * No-allocation variant of sparse_attn_fwd.  The pages have no counterpart;
 * it exists for callers that cannot allocate device memory: programs that
 * reserve all their device memory up front in a pool of their own and must
 * not call cudaMalloc afterwards (it can block the host, stall other work on
 * the device, and fail under memory pressure mid-request).  sparse_attn_fwd
 * allocates a status word on its first call on a device and reads the block
 * mask from device memory the caller allocated; this call does neither.
 *
 * Arguments as sparse_attn_fwd, except that `mask` holds the HOST arrays
 * returned by sparse_attn_build_block_mask, and that only the causal forms are
 * taken (causal == 1 with window, sinks, stride and n_global; causal == 0,
 * area > 0 or summary > 0 give SA_ERR_UNSUPPORTED).  The mask is checked on
 * the host before any device work, as for sparse_attn_fwd_host
 * (SA_ERR_INVALID_ARG).  Its scratch, the kernel's status word and a device
 * copy of the mask, lives in one static device array of
 * SA_NOALLOC_SCRATCH_BYTES that the library holds on every GPU that loads it
 * until the process exits.  A mask that does not fit (with 256 bytes for the
 * status word, 4 T + 5 T^2 bytes for T tiles per side: T <= 457) is rejected
 * with SA_ERR_SCRATCH_TOO_SMALL before any device work.  The wait limit and
 * the skip-Q-load hook of sparse_attn_set_debug apply here too.
 *
 * The first call on a device looks up the array's device address with that
 * device current.  Every call clears the status word, copies the mask from
 * host memory, launches on `stream`, copies the status word back into host
 * memory and waits for the stream, then returns the device status
 * (SA_ERR_DEVICE_TIMEOUT if a bounded wait expired): a call therefore cannot
 * be made while `stream` is being captured into a CUDA graph.  All calls
 * share the array and it keeps the last call's contents; calls whose kernels
 * overlap on the GPU race on it (calls from several host threads are
 * serialised per device).  Calls no cudaMalloc, cudaFree or other allocating
 * routine.
 */
#define SA_NOALLOC_SCRATCH_BYTES (1u << 20)
int sparse_attn_fwd_noalloc(const void* Q, const void* K, const void* V, const sa_block_mask* mask_host,
                            const sa_pattern* pattern, const sa_shape* shape, float scale, void* O, float* LSE,
                            void* stream);

/*
 * Transpose a compiled block mask: for every kv tile c, the ascending list of
 * query tiles whose list holds c, with the same full flags.  The result uses
 * the sa_block_mask fields with rows and columns swapped: kv_count[c] is the
 * number of query tiles listed for kv tile c, kv_index[c*T + e] the e-th of
 * them (-1 after the last), kv_full[c*T + e] its flag (0 after the last).
 * Host-only; `rows` as written by sparse_attn_build_block_mask, `cols` with
 * caller-owned host arrays of capacity cols->n_q_tiles x cols->n_kv_tiles, both
 * at least T (else SA_ERR_BUFFER_TOO_SMALL).  SA_ERR_INVALID_ARG for null
 * arguments or an inconsistent input (counts or indices out of range).
 */
int sparse_attn_transpose_block_mask(const sa_block_mask* rows, sa_block_mask* cols);

/* Device workspace bytes that sparse_attn_bwd needs for `shape`:
 * 4 B * Hq * N (LSE in base 2) + 4 B * Hq * N (row term) + 4 B * Hq * N * D
 * (fp32 dQ accumulator), each rounded up to 256 bytes. */
int sparse_attn_bwd_workspace(const sa_shape* shape, size_t* bytes);

/*
 * Backward pass: the gradients dQ, dK, dV of the attention computed by
 * sparse_attn_fwd, for an upstream gradient dO.  The pages print no backward
 * pass; this is the chain rule through the masked softmax of the
 * "Sparse-трансформеры" page, section "Как это выглядит в коде": with P the
 * softmax weights of each query over its allowed keys,
 *   dV = P^T dO,  dS = P * (dO V^T - rowsum(dO * O)),
 *   dQ = scale * dS K,  dK = scale * dS^T Q,
 * and for grouped heads dK, dV summed over the query heads of the group.
 *
 * All tensors in DEVICE memory, contiguous, 16-byte aligned:
 *   Q, O, dO, dQ [B, Hq, N, D] bf16;  K, V, dK, dV [B, Hkv, N, D] bf16;
 *   LSE [B, Hq, N] fp32 as written by sparse_attn_fwd (natural log).
 *   mask_t     the TRANSPOSED block mask (sparse_attn_transpose_block_mask of
 *              the pattern's mask) with its arrays in device memory (checked as
 *              for sparse_attn_fwd); block 128
 *   pattern    the pattern the mask was compiled from (partial tiles are
 *              masked element by element from it)
 *   workspace  device memory of at least sparse_attn_bwd_workspace bytes,
 *              256-byte aligned; caller-owned, contents need not be preserved
 * Launches four kernels on `stream` (work items, row sums, the main kernel,
 * dQ conversion) and returns without waiting; the
 * workspace must not be reused until they finish.  The caller owns every
 * buffer.  Errors as sparse_attn_fwd, plus SA_ERR_UNSUPPORTED for a mask block
 * other than 128 and SA_ERR_BUFFER_TOO_SMALL for a short workspace; a bounded
 * wait that expires inside the kernel sets the status word that
 * sparse_attn_check_device reports.
 */
int sparse_attn_bwd(const void* Q, const void* K, const void* V, const void* O, const float* LSE, const void* dO,
                    const sa_block_mask* mask_t, const sa_pattern* pattern, const sa_shape* shape, float scale,
                    void* dQ, void* dK, void* dV, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward pass with a pattern per query head, the gradients of
 * sparse_attn_fwd_heads: query head h under patterns[head_pattern[h]], whose
 * TRANSPOSED block mask (device arrays, block 128) is masks_t[head_pattern[h]];
 * for grouped heads dK, dV sum the heads of the group, each under its own
 * pattern.  n_patterns 1 .. 8, head_pattern [Hq] (host), Hq <= 256; other
 * arguments, layouts and errors as sparse_attn_bwd (SA_ERR_INVALID_ARG for a
 * null head table, a count out of range or an index outside [0, n_patterns)).
 */
int sparse_attn_bwd_heads(const void* Q, const void* K, const void* V, const void* O, const float* LSE,
                          const void* dO, const sa_block_mask* masks_t, const sa_pattern* patterns, int32_t n_patterns,
                          const int32_t* head_pattern, const sa_shape* shape, float scale, void* dQ, void* dK,
                          void* dV, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Stride-aware path for causal patterns with a stride s (every s-th prior
 * token): in token order those pairs touch every tile below the diagonal once
 * per row.  The plan splits the pattern into
 *   pass 1  the pattern without its stride, in token order, and
 *   pass 2  the stride pairs that pass 1 does not admit, on tokens grouped by
 *           residue (position P = (t mod s) * n + floor(t / s), n = N / s),
 *           where they form dense tiles along the diagonal,
 * and sparse_attn_fwd_stride merges the two partial softmaxes exactly.  Needs
 * causal == 1, stride > 0, area == 0, and N a multiple of the stride (else
 * SA_ERR_UNSUPPORTED).  Host-only; pass1 and pass2 hold caller-owned host
 * arrays of capacity T x T each (T = ceil(N / block)), as for
 * sparse_attn_build_block_mask.
 */
int sparse_attn_stride_plan(const sa_pattern* pattern, int64_t N, int32_t block, sa_block_mask* pass1,
                            sa_block_mask* pass2);

/* Device workspace bytes that sparse_attn_fwd_stride needs: grouped copies of
 * Q, K, V, pass 2's O (bf16), and both passes' LSE (fp32), each rounded up to
 * 256 bytes. */
int sparse_attn_fwd_stride_workspace(const sa_shape* shape, size_t* bytes);

/*
 * The forward pass by the stride-aware path: results as sparse_attn_fwd with
 * `pattern` (O, LSE of the whole pattern).  pass1 and pass2 are the plan's
 * masks with their arrays in DEVICE memory; workspace is device memory of at
 * least sparse_attn_fwd_stride_workspace bytes, 256-byte aligned.  Launches
 * three grouping copies, the two passes and the merge on `stream`; returns
 * without waiting.  Errors as sparse_attn_fwd, plus SA_ERR_UNSUPPORTED for a
 * pattern the plan does not take and SA_ERR_BUFFER_TOO_SMALL for a short
 * workspace.
 */
int sparse_attn_fwd_stride(const void* Q, const void* K, const void* V, const sa_block_mask* pass1,
                           const sa_block_mask* pass2, const sa_pattern* pattern, const sa_shape* shape, float scale,
                           void* O, float* LSE, void* workspace, size_t workspace_bytes, void* stream);

const char* sparse_attn_status_string(int status);

/* ABI version: major * 10000 + minor * 100 + patch. */
int32_t sparse_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_H */
