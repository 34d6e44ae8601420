/*
 * bd.h -- C ABI of libbd: one denoising step of block-diffusion decoding
 * (Fast-dLLM v2) on an NVIDIA B200 (sm_100a).
 *
 * Method sources, cited by page title and section:
 *   [N1] "Fast-dLLM v2: Efficient Block-Diffusion LLM", paper notes
 *        (papernotes.org), "Overall framework" and "Key designs" 1-4.
 *   [N2] Fast-dLLM (v1) article (senqingzn.com), "Core techniques" item 2,
 *        confidence-aware parallel decoding.
 *   [N3] Fast-dLLM v2 abstract (hyper.ai, arXiv 2509.26328): training with
 *        complementary masks.
 *   [N4] "Fast-dLLM v2: 2.5x inference speedup" (aigc.bar), "Acceleration
 *        engine" items 1 (hierarchical cache) and 2 (parallel decoding).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - A block is BD_BLOCK = 32 tokens.  Tensors are dense, row-major, in the
 *   element type named by a bd_dtype (fp32, or bf16 with fp32 arithmetic).
 * - Pointers marked "device" must be CUDA device memory of the current
 *   device; "host" pointers are read on the host during the call only.
 * - The library allocates nothing and keeps no state between calls: the
 *   caller owns every buffer, the KV cache and the scratch workspace.  Ask
 *   for the workspace size with the matching *_workspace_size call.
 * - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *   stream) and the call returns without synchronising.
 * - Every entry point returns a bd_status.  Argument errors are found on the
 *   host before anything is launched (nothing is enqueued then).  BD_ERR_CUDA
 *   reports a launch failure; the CUDA error string is then available from
 *   bd_last_cuda_error_string().  Nothing throws across this boundary.
 * - Calls on the same stream are ordered; calls that share a workspace or a
 *   cache must not run concurrently on different streams.
 */
#ifndef BD_H_
#define BD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BD_BLOCK 32

#if defined(__GNUC__)
#define BD_API __attribute__((visibility("default")))
#else
#define BD_API
#endif

typedef enum {
  BD_OK = 0,
  BD_ERR_INVALID_ARG = -1, /* null pointer, bad size or shape            */
  BD_ERR_UNSUPPORTED = -2, /* shape or dtype this build does not handle  */
  BD_ERR_CAPACITY = -3,    /* KV cache page table / pages exhausted      */
  BD_ERR_WORKSPACE = -4,   /* workspace missing or too small             */
  BD_ERR_CUDA = -5         /* a CUDA launch or runtime call failed       */
} bd_status;

typedef enum { BD_F32 = 0, BD_BF16 = 1 } bd_dtype;

/* Attention geometry.  Query head h reads KV head h / (n_heads_q /
 * n_heads_kv) (contiguous groups).  head_dim is 64 or 128.  rope_theta is
 * the RoPE base: pair (j, j + d/2) rotates by pos * rope_theta^(-2j/d). */
typedef struct {
  int32_t n_heads_q;
  int32_t n_heads_kv;
  int32_t head_dim;
  int32_t dtype;     /* bd_dtype of q, k, v, cache pages and outputs */
  double rope_theta;
} bd_attn_shape;

/* Block-level KV cache ([N1] key design 3; [N4] item 1): per sequence, the
 * K and V of every finished block, each block stored as one page.  Keys are
 * stored already rotated (RoPE at their absolute positions).
 *
 *   pages       device, [n_pages][2][n_heads_kv][32][head_dim] of dtype;
 *               index 0 of the second axis is K, 1 is V.
 *   page_table  device, [batch][max_blocks] int32: physical page of logical
 *               block b of sequence s (caller-assigned, distinct pages).
 *   n_blocks    device, [batch] int32: finished blocks per sequence.
 *   *_host      host mirrors of page_table and n_blocks with the same
 *               contents; the library reads them for validation and launch
 *               sizing and keeps n_blocks_host in step on commit.
 */
typedef struct {
  void* pages;
  int64_t n_pages;
  int32_t* page_table;
  const int32_t* page_table_host;
  int32_t* n_blocks;
  int32_t* n_blocks_host;
  int32_t batch;
  int32_t max_blocks;
} bd_kv_cache;

/* bd_cache_commit -- append finished blocks to the block-level KV cache.
 *
 * [N1] key design 3 / [N4] item 1: once a block is fully decoded its K/V are
 * kept as read-only context for every later block, exactly like an
 * autoregressive KV cache.
 *
 *   k, v      device, [n_seqs][32 * n_new_blocks][n_heads_kv][head_dim]
 *             (k before RoPE).
 *   seq_ids   host, [n_seqs] distinct sequence indices in [0, batch).
 * For each listed sequence s with P = 32 * n_blocks_host[s], token t of the
 * input is written, k rotated at absolute position P + t, into page
 * page_table[s][n_blocks_host[s] + t / 32], row t % 32; then n_blocks (device
 * and host) grows by n_new_blocks.  Errors: BD_ERR_CAPACITY when
 * n_blocks_host[s] + n_new_blocks > max_blocks; BD_ERR_INVALID_ARG for a
 * page id outside [0, n_pages) or a repeated / out-of-range sequence. */
BD_API int bd_cache_commit(const bd_attn_shape* shape, bd_kv_cache* cache,
                    const void* k, const void* v, const int32_t* seq_ids,
                    int32_t n_seqs, int32_t n_new_blocks, void* stream);

/* bd_block_attn -- attention of the current block over the cache.
 *
 * [N1] overall framework and key design 3; [N4] "block-internal parallel,
 * block-causal": every query of the current 32-token block sees all cached
 * keys of its sequence and all 32 keys of its own block, unmasked.
 *
 *   q      device, [batch][32][n_heads_q][head_dim], before RoPE
 *   k_blk  device, [batch][32][n_heads_kv][head_dim], before RoPE
 *   v_blk  device, [batch][32][n_heads_kv][head_dim]
 *   out    device, [batch][32][n_heads_q][head_dim], written
 * q and k_blk are rotated at positions P..P+31 (P = 32 * n_blocks[s]);
 * out = softmax(q K^T / sqrt(head_dim)) V over [cached keys ; block keys].
 * q, k_blk, v_blk and out are 16-byte aligned (BD_ERR_INVALID_ARG
 * otherwise).  batch is cache->batch.  Workspace: bd_block_attn_workspace_size() bytes,
 * 256-byte aligned; its size depends on n_blocks_host, so ask again after
 * the cache grows. */
BD_API int bd_block_attn_workspace_size(const bd_attn_shape* shape,
                                 const bd_kv_cache* cache, size_t* bytes);
BD_API int bd_block_attn(const bd_attn_shape* shape, const bd_kv_cache* cache,
                  const void* q, const void* k_blk, const void* v_blk,
                  void* out, void* workspace, size_t workspace_bytes,
                  void* stream);

/* bd_confidence_select -- confidence-aware parallel unmask of one step.
 *
 * [N1] key designs 2-4, [N2] item 2, [N4] item 2.  For every masked
 * position i of each sequence (bit i of masked_bits[s]):
 *   row    = hidden row i-1 of the block, or h_prev[s] for i = 0 (token
 *            shift, key design 2);
 *   l      = row . w_lm[v] for every vocab entry v (logits never stored);
 *   token  = argmax_v l (lowest v on ties); p_max = 1 / sum_v exp(l - max l).
 * Candidates are the masked positions of the lowest sub-block of
 * `sub_block` positions that still holds a masked position (key design 4).
 * Every candidate with p_max > tau is unmasked; if there is none, the single
 * candidate with the largest p_max is (lowest position on ties).
 *
 *   dtype        element type of h, h_prev and w_lm
 *   h            device, [batch][32][hidden]
 *   h_prev       device, [batch][hidden]
 *   w_lm         device, [vocab][hidden]
 *   masked_bits  device, [batch] uint32; not modified
 *   tokens       device, [batch][32] int32; unmasked positions receive
 *                their token, all others are left as they are
 *   unmask_bits  device, [batch] uint32 out: positions unmasked this step
 *   pmax_out     device, [batch][32] float or NULL: p_max per masked
 *                position, NaN elsewhere
 *   argmax_out   device, [batch][32] int32 or NULL: token per masked
 *                position, -1 elsewhere
 * sub_block must divide 32; 0 <= tau; hidden % 8 == 0; h, h_prev and w_lm
 * 16-byte aligned.  Workspace: bd_confidence_select_workspace_size() bytes,
 * 256-byte aligned, its first 256 bytes zero before the first call that
 * uses it (cudaMemset once when it is allocated): the library keeps a
 * status word and an arrival counter there, which every call leaves ready
 * for the next, so the caller must not write to them between calls, nor
 * use one workspace in two calls that may run at the same time.  bf16 runs
 * the LM head on the tensor cores (tcgen05): if one of its bounded waits
 * ever gives up (it never should), the call reports "no decision" for the
 * whole batch: unmask_bits 0, p_max NaN and argmax -2. */
BD_API int bd_confidence_select_workspace_size(int32_t dtype, int32_t batch,
                                        int32_t hidden, int32_t vocab,
                                        size_t* bytes);
BD_API int bd_confidence_select(int32_t dtype, int32_t batch, int32_t hidden,
                         int32_t vocab, const void* h, const void* h_prev,
                         const void* w_lm, const uint32_t* masked_bits,
                         float tau, int32_t sub_block, int32_t* tokens,
                         uint32_t* unmask_bits, float* pmax_out,
                         int32_t* argmax_out, void* workspace,
                         size_t workspace_bytes, void* stream);

/* bd_confidence_select_active -- bd_confidence_select that scores only the
 * candidates of the unmask rule.
 *
 * The rule picks only among the masked positions of the lowest sub-block
 * that still has one ([N1] key design 4: the sub-block sets the decoding
 * granularity inside the block), so scoring the other masked positions
 * decides nothing.  This call computes the LM-head statistics for those
 * candidates alone (at most sub_block positions per sequence instead of up
 * to 32).  Same arguments, workspace and errors as bd_confidence_select;
 * tokens and unmask_bits are the same; pmax_out / argmax_out hold NaN / -1
 * at every position that is not a candidate. */
BD_API int bd_confidence_select_active(int32_t dtype, int32_t batch, int32_t hidden,
                                int32_t vocab, const void* h, const void* h_prev,
                                const void* w_lm, const uint32_t* masked_bits,
                                float tau, int32_t sub_block, int32_t* tokens,
                                uint32_t* unmask_bits, float* pmax_out,
                                int32_t* argmax_out, void* workspace,
                                size_t workspace_bytes, void* stream);

/* bd_masked_ce -- masked-token cross-entropy of training, logits on chip.
 *
 * [N1] key design 2, the L_block equation with the shifted label: in each of
 * n_seqs training sequences of seq_len positions (the noisy stream x_t),
 * every position i >= 1 whose token is [MASK] contributes
 *     -log softmax(W h_{i-1})[x_0^i]  =  max l + log sum exp(l - max) - l_y,
 * l = W h_{i-1}; position 0 of a sequence has no previous row and is not
 * scored.  The expectation of the equation is left to the caller.
 *
 *   h            device, [n_seqs][seq_len][hidden]: final hidden rows of x_t
 *   w_lm         device, [vocab][hidden]
 *   targets      device, [n_seqs][seq_len] int32: the clean tokens x_0
 *   masked_bits  device, [n_seqs][seq_len / 32] uint32: bit i % 32 of word
 *                i / 32 set = position i is [MASK] in x_t
 *   loss_out     device, [n_seqs][seq_len] float or NULL: the loss at every
 *                scored position, NaN elsewhere
 *   loss_sum     device, [1] float: the sum over the scored positions (added
 *                in a fixed order: the same inputs give the same bits)
 *   n_scored     device, [1] int32 or NULL: the number of scored positions
 * seq_len % 32 == 0; hidden % 8 == 0; h and w_lm 16-byte aligned.  A target
 * outside [0, vocab) gives a NaN loss.  Workspace:
 * bd_masked_ce_workspace_size() bytes, 256-byte aligned.  bf16 with up to
 * 148 x 256 positions runs the LM head on the tensor cores; if one of its
 * bounded waits ever gives up, every loss is NaN. */
BD_API int bd_masked_ce_workspace_size(int32_t dtype, int32_t n_seqs,
                                int32_t seq_len, int32_t hidden, int32_t vocab,
                                size_t* bytes);
BD_API int bd_masked_ce(int32_t dtype, int32_t n_seqs, int32_t seq_len,
                 int32_t hidden, int32_t vocab, const void* h,
                 const void* w_lm, const int32_t* targets,
                 const uint32_t* masked_bits, float* loss_out, float* loss_sum,
                 int32_t* n_scored, void* workspace, size_t workspace_bytes,
                 void* stream);

/* bd_confidence_select_noalloc -- bd_confidence_select without a workspace.
 *
 * The method's description has no counterpart to this call: it exists for
 * callers that cannot allocate device memory when they run the step, such
 * as a plugin that its host application hands only input and output
 * buffers, code running while a framework's caching allocator owns the whole
 * device, or a latency-bound loop that must not pay cudaMalloc's implicit
 * device synchronisation.
 *
 * Same arguments, results and errors as bd_confidence_select, minus the
 * workspace: the step's scratch lives in one fixed array of
 * BD_NOALLOC_SCRATCH_BYTES that the library keeps in device memory on every
 * GPU where it is loaded, until the process exits.  A step whose scratch
 * would exceed it (roughly batch * 32 rows * hidden elements plus 12 bytes
 * per row and SM) is refused with BD_ERR_WORKSPACE before anything runs: in
 * bf16 on a 148-SM B200 that is a batch above 24 at hidden 3584, above 48
 * at hidden 1536.  The call
 * allocates nothing.  Its first call on a device looks the array's device
 * address up (cudaGetSymbolAddress) with that device current and keeps it
 * for the life of the process: make that first call before any stream
 * capture on the device, and do not use this call after a cudaDeviceReset.
 * Every call on a device shares the one array.  Each call first clears the
 * array's 16-byte header on `stream` (cudaMemsetAsync: the single-kernel
 * path counts CTA arrivals and vocab tiles there and needs them zero at the
 * start); the rest of the array holds the last call's packed rows and
 * partials, which the next call overwrites before it reads them.  Calls
 * whose work overlaps on the GPU -- different streams, or different host
 * threads on one device -- race on the array and must be serialised by the
 * caller. */
#define BD_NOALLOC_SCRATCH_BYTES (8u << 20)
BD_API int bd_confidence_select_noalloc(int32_t dtype, int32_t batch, int32_t hidden,
                                        int32_t vocab, const void* h, const void* h_prev,
                                        const void* w_lm, const uint32_t* masked_bits,
                                        float tau, int32_t sub_block, int32_t* tokens,
                                        uint32_t* unmask_bits, float* pmax_out,
                                        int32_t* argmax_out, void* stream);

/* bd_block_mask_attn -- attention of the training forward under the 2L x 2L
 * complementary mask ([N1] key design 2).
 *
 * Each of the n_seqs entries (one per sample and mask view) is the noisy
 * stream x_t (rows 0..L-1) followed by the clean stream x_0 (rows L..2L-1).
 * With blk(i) = (i mod L) / block: a noisy query sees the noisy keys of its
 * own block and the clean keys of earlier blocks; a clean query sees the
 * clean keys of its own and earlier blocks; no clean query sees a noisy key.
 *
 *   q     device, [n_seqs][2L][n_heads_q][head_dim] (already rotated)
 *   k, v  device, [n_seqs][2L][n_heads_kv][head_dim]
 *   out   device, [n_seqs][2L][n_heads_q][head_dim], written
 * block must divide L; shape->rope_theta is ignored. */
BD_API int bd_block_mask_attn(const bd_attn_shape* shape, const void* q,
                       const void* k, const void* v, void* out,
                       int32_t n_seqs, int32_t L, int32_t block, void* stream);

/* bd_block_mask_attn_views -- bd_block_mask_attn for a batch whose entries
 * come in groups of `views` consecutive entries that are views of one
 * training sample ([N1] key design 2: the complementary masks m and 1 - m
 * of one sample are two views of it, [N3]).  The views of a sample differ
 * only in their noisy stream; their clean halves (rows L..2L-1 of q, k and
 * v) must be equal, and the caller guarantees that.  A clean query sees
 * clean keys only, so the clean rows of the output are equal across the
 * views: the tensor-core path computes them once per sample, from its first
 * view, and writes them into every view's rows (with views = 2 that is a
 * quarter of the pairs of the plain call).  Arguments, layouts and errors as
 * bd_block_mask_attn, plus:
 *   views  >= 1 and dividing n_seqs (else BD_ERR_INVALID_ARG); views = 1 is
 *          the plain call.
 * If the clean halves of a sample's views differ, views other than the
 * first receive the first view's clean rows.  Other shapes than the
 * tensor-core kernel's (bf16, head_dim 128, L a multiple of 128) compute
 * every view's rows from its own inputs. */
BD_API int bd_block_mask_attn_views(const bd_attn_shape* shape, const void* q,
                                    const void* k, const void* v, void* out,
                                    int32_t n_seqs, int32_t views, int32_t L,
                                    int32_t block, void* stream);

/* bd_eval_exp2 -- diagnostic: the library's exponential approximations.
 *
 * No counterpart in the method: the attention softmax and the LM-head
 * statistics evaluate part of their exponentials 2^x with a polynomial on
 * the FMA pipe (relative error below 2.7e-6 for -126 <= x <= 0) and the rest
 * with the hardware approximation; this call evaluates them on given
 * arguments so that a test can check those bounds on the device.
 *   x       device, [n] float arguments
 *   y_poly  device, [n] out: the scalar polynomial
 *   y_pair  device, [n] out: the paired (two-lane) polynomial, on the pairs
 *           (x[2i], x[2i+1])
 *   y_mufu  device, [n] out: the hardware approximation (ex2.approx.ftz)
 * BD_ERR_INVALID_ARG for a null pointer or n < 0. */
BD_API int bd_eval_exp2(const float* x, float* y_poly, float* y_pair, float* y_mufu,
                        int32_t n, void* stream);

/* bd_device_check_status -- diagnostic: the device-side index checks.
 *
 * No counterpart in the method.  The library built with BD_DEVICE_CHECKS
 * defined (libbd_checks.so; `python -m decoding_bd_block_b200.build`
 * builds it beside libbd.so) checks, inside its kernels, the indices it reads
 * from device memory: cache page ids (commit, block attention), packed-row
 * indices (confidence select) and target ids (masked CE).  A failed check
 * skips the access as the normal build does (zeros are read, nothing is
 * written) and records {code, detail}: the first failure since the last
 * reset wins.  This call copies that record to the host (it waits for the
 * device), and clears it when `reset` is nonzero.
 *   code    host, out: 0 none, 1 page id outside [0, n_pages), 2 packed-row
 *           index out of range, 3 target id outside [0, vocab)
 *   detail  host, out: the offending value
 * Returns BD_ERR_UNSUPPORTED in a build without the checks. */
BD_API int bd_device_check_status(int32_t* code, int32_t* detail, int32_t reset);

/* Human-readable name of a bd_status value. */
BD_API const char* bd_status_string(int status);
/* Text of the last CUDA error seen by a call of this thread (or ""). */
BD_API const char* bd_last_cuda_error_string(void);
/* Number of CUDA kernels this library has enqueued in this process so far
 * (all threads).  A diagnostic for measuring launches per step. */
BD_API long long bd_kernel_launches(void);

#ifdef __cplusplus
}
#endif
#endif /* BD_H_ */
