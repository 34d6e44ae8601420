// C-ABI entry points of libbd: host-side validation, workspace planning and
// dispatch to the kernels.  Nothing here allocates device memory.
#include <atomic>
#include <cmath>
#include <cstring>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "bd_common.cuh"
#include "mask_attn.cuh"

namespace bd {
static std::atomic<long long> g_launches{0};
void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

void rope_freq_table(int d, double theta, RopeFreq* f) {
  for (int j = 0; j < 64; ++j)
    f->inv[j] = j < d / 2 ? std::pow(theta, -2.0 * j / static_cast<double>(d)) : 0.0;
}
}  // namespace bd

namespace {

// A profiler-visible range named after the entry point, for the duration of
// the call (NVTX: a no-op unless a tool such as Nsight is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

thread_local char g_cuda_err[256] = "";

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return BD_OK;
  std::strncpy(g_cuda_err, cudaGetErrorString(e), sizeof(g_cuda_err) - 1);
  g_cuda_err[sizeof(g_cuda_err) - 1] = '\0';
  return BD_ERR_CUDA;
}

int check_shape(const bd_attn_shape* sh) {
  if (!sh) return BD_ERR_INVALID_ARG;
  if (sh->n_heads_q <= 0 || sh->n_heads_kv <= 0 || sh->n_heads_q % sh->n_heads_kv != 0)
    return BD_ERR_INVALID_ARG;
  if (sh->dtype != BD_F32 && sh->dtype != BD_BF16) return BD_ERR_UNSUPPORTED;
  if (sh->head_dim != 64 && sh->head_dim != 128) return BD_ERR_UNSUPPORTED;
  if (sh->n_heads_q > 1024) return BD_ERR_UNSUPPORTED;
  return BD_OK;
}

int check_cache(const bd_attn_shape* sh, const bd_kv_cache* c) {
  if (!c || !c->pages || !c->page_table || !c->page_table_host || !c->n_blocks ||
      !c->n_blocks_host)
    return BD_ERR_INVALID_ARG;
  if (c->batch <= 0 || c->batch > 65535 || c->max_blocks <= 0 || c->n_pages <= 0)
    return BD_ERR_INVALID_ARG;
  if (!(sh->rope_theta > 0.0)) return BD_ERR_INVALID_ARG;
  for (int s = 0; s < c->batch; ++s) {
    const int nb = c->n_blocks_host[s];
    if (nb < 0 || nb > c->max_blocks) return BD_ERR_INVALID_ARG;
    for (int b = 0; b < nb; ++b) {
      const int pg = c->page_table_host[static_cast<size_t>(s) * c->max_blocks + b];
      if (pg < 0 || pg >= c->n_pages) return BD_ERR_INVALID_ARG;
    }
  }
  return BD_OK;
}

}  // namespace

namespace bd {
int report_cuda_error(cudaError_t e) { return cuda_status(e); }
}  // namespace bd

extern "C" {

const char* bd_status_string(int status) {
  switch (status) {
    case BD_OK: return "ok";
    case BD_ERR_INVALID_ARG: return "invalid argument";
    case BD_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case BD_ERR_CAPACITY: return "KV cache capacity exceeded";
    case BD_ERR_WORKSPACE: return "workspace missing or too small";
    case BD_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

const char* bd_last_cuda_error_string(void) { return g_cuda_err; }

long long bd_kernel_launches(void) { return bd::g_launches.load(std::memory_order_relaxed); }

int bd_device_check_status(int32_t* code, int32_t* detail, int32_t reset) {
#ifdef BD_DEVICE_CHECKS
  if (!code || !detail) return BD_ERR_INVALID_ARG;
  *code = 0;
  *detail = 0;
  cudaError_t (*const units[])(int*, bool) = {bd::check_word_commit, bd::check_word_attn_tc,
                                              bd::check_word_attn_simt, bd::check_word_select,
                                              bd::check_word_ce};
  for (auto unit : units) {
    int w[2] = {0, 0};
    const int st = cuda_status(unit(w, reset != 0));
    if (st) return st;
    if (*code == 0 && w[0] != 0) {
      *code = w[0];
      *detail = w[1];
    }
  }
  return BD_OK;
#else
  (void)code;
  (void)detail;
  (void)reset;
  return BD_ERR_UNSUPPORTED;
#endif
}

int bd_cache_commit(const bd_attn_shape* sh, bd_kv_cache* c, const void* k, const void* v,
                    const int32_t* seq_ids, int32_t n_seqs, int32_t n_new_blocks, void* stream) {
  NvtxRange nvtx_range("bd_cache_commit");
  int st = check_shape(sh);
  if (st) return st;
  if ((st = check_cache(sh, c))) return st;
  if (!k || !v || !seq_ids || n_seqs <= 0 || n_seqs > c->batch || n_new_blocks <= 0 ||
      n_new_blocks > 65535 / bd::kBlock)
    return BD_ERR_INVALID_ARG;
  std::vector<char> seen(c->batch, 0);
  for (int i = 0; i < n_seqs; ++i) {
    const int s = seq_ids[i];
    if (s < 0 || s >= c->batch || seen[s]) return BD_ERR_INVALID_ARG;
    seen[s] = 1;
    if (c->n_blocks_host[s] + static_cast<long long>(n_new_blocks) > c->max_blocks)
      return BD_ERR_CAPACITY;
  }
  // The new pages must be valid, distinct, and not hold a committed block.
  std::vector<char> used(static_cast<size_t>(c->n_pages), 0);
  for (int s = 0; s < c->batch; ++s)
    for (int b = 0; b < c->n_blocks_host[s]; ++b)
      used[c->page_table_host[static_cast<size_t>(s) * c->max_blocks + b]] = 1;
  for (int i = 0; i < n_seqs; ++i) {
    const int s = seq_ids[i];
    for (int b = 0; b < n_new_blocks; ++b) {
      const int pg =
          c->page_table_host[static_cast<size_t>(s) * c->max_blocks + c->n_blocks_host[s] + b];
      if (pg < 0 || pg >= c->n_pages) return BD_ERR_INVALID_ARG;
      if (used[pg]) return BD_ERR_INVALID_ARG;
      used[pg] = 1;
    }
  }
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  for (int i0 = 0; i0 < n_seqs; i0 += 256) {
    bd::CommitArgs a{};
    a.n_seqs = n_seqs - i0 < 256 ? n_seqs - i0 : 256;
    a.n_new_blocks = n_new_blocks;
    for (int i = 0; i < a.n_seqs; ++i) {
      a.seq_ids[i] = seq_ids[i0 + i];
      a.first_block[i] = c->n_blocks_host[seq_ids[i0 + i]];
    }
    const size_t tok = static_cast<size_t>(bd::kBlock) * n_new_blocks * sh->n_heads_kv *
                       sh->head_dim * (sh->dtype == BD_BF16 ? 2 : 4);
    const char* kk = static_cast<const char*>(k) + tok * i0;
    const char* vv = static_cast<const char*>(v) + tok * i0;
    st = cuda_status(bd::launch_cache_commit(*sh, *c, kk, vv, a, strm));
    if (st) return st;
  }
  for (int i = 0; i < n_seqs; ++i) c->n_blocks_host[seq_ids[i]] += n_new_blocks;
  return BD_OK;
}

int bd_block_attn_workspace_size(const bd_attn_shape* sh, const bd_kv_cache* c, size_t* bytes) {
  int st = check_shape(sh);
  if (st) return st;
  if (!bytes) return BD_ERR_INVALID_ARG;
  if ((st = check_cache(sh, c))) return st;
  *bytes = bd::plan_block_attn(*sh, *c).total;
  return BD_OK;
}

int bd_block_attn(const bd_attn_shape* sh, const bd_kv_cache* c, const void* q, const void* k,
                  const void* v, void* out, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("bd_block_attn");
  int st = check_shape(sh);
  if (st) return st;
  if ((st = check_cache(sh, c))) return st;
  if (!q || !k || !v || !out) return BD_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, static_cast<const void*>(out)})
    if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0) return BD_ERR_INVALID_ARG;
  const bd::AttnPlan p = bd::plan_block_attn(*sh, *c);
  if (p.total > 0 && (!ws || ws_bytes < p.total)) return BD_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return BD_ERR_WORKSPACE;
  return cuda_status(
      bd::launch_block_attn(*sh, *c, p, q, k, v, out, ws, static_cast<cudaStream_t>(stream)));
}

int bd_confidence_select_workspace_size(int32_t dtype, int32_t batch, int32_t hidden,
                                        int32_t vocab, size_t* bytes) {
  if (!bytes || batch <= 0 || batch > 65535 || hidden <= 0 || vocab <= 0)
    return BD_ERR_INVALID_ARG;
  if (dtype != BD_F32 && dtype != BD_BF16) return BD_ERR_UNSUPPORTED;
  *bytes = bd::plan_confidence_select(dtype, batch, hidden, vocab).total;
  return BD_OK;
}

namespace {
int confidence_select(int32_t dtype, int32_t batch, int32_t hidden, int32_t vocab, const void* h,
                      const void* h_prev, const void* w, const uint32_t* masked_bits, float tau,
                      int32_t sub_block, int32_t* tokens, uint32_t* unmask_bits, float* pmax_out,
                      int32_t* argmax_out, void* ws, size_t ws_bytes, void* stream, int active) {
  if (batch <= 0 || batch > 65535 || hidden <= 0 || vocab <= 0) return BD_ERR_INVALID_ARG;
  if (dtype != BD_F32 && dtype != BD_BF16) return BD_ERR_UNSUPPORTED;
  if (hidden % 8 != 0) return BD_ERR_UNSUPPORTED;
  if (!h || !h_prev || !w || !masked_bits || !tokens || !unmask_bits) return BD_ERR_INVALID_ARG;
  // rows are copied in 16-byte vectors and W is read by TMA
  if ((reinterpret_cast<uintptr_t>(h) | reinterpret_cast<uintptr_t>(h_prev) |
       reinterpret_cast<uintptr_t>(w)) % 16 != 0)
    return BD_ERR_INVALID_ARG;
  if (sub_block <= 0 || sub_block > bd::kBlock || bd::kBlock % sub_block != 0)
    return BD_ERR_INVALID_ARG;
  if (!(tau >= 0.f)) return BD_ERR_INVALID_ARG;
  const bd::SelectPlan p = bd::plan_confidence_select(dtype, batch, hidden, vocab);
  if (!ws || ws_bytes < p.total) return BD_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return BD_ERR_WORKSPACE;
  return cuda_status(bd::launch_confidence_select(dtype, batch, hidden, vocab, p, h, h_prev, w,
                                                  masked_bits, tau, sub_block, tokens,
                                                  unmask_bits, pmax_out, argmax_out, ws,
                                                  static_cast<cudaStream_t>(stream), active));
}
}  // namespace

int bd_confidence_select(int32_t dtype, int32_t batch, int32_t hidden, int32_t vocab,
                         const void* h, const void* h_prev, const void* w,
                         const uint32_t* masked_bits, float tau, int32_t sub_block,
                         int32_t* tokens, uint32_t* unmask_bits, float* pmax_out,
                         int32_t* argmax_out, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("bd_confidence_select");
  return confidence_select(dtype, batch, hidden, vocab, h, h_prev, w, masked_bits, tau, sub_block,
                           tokens, unmask_bits, pmax_out, argmax_out, ws, ws_bytes, stream, 0);
}

int bd_confidence_select_active(int32_t dtype, int32_t batch, int32_t hidden, int32_t vocab,
                                const void* h, const void* h_prev, const void* w,
                                const uint32_t* masked_bits, float tau, int32_t sub_block,
                                int32_t* tokens, uint32_t* unmask_bits, float* pmax_out,
                                int32_t* argmax_out, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("bd_confidence_select_active");
  return confidence_select(dtype, batch, hidden, vocab, h, h_prev, w, masked_bits, tau, sub_block,
                           tokens, unmask_bits, pmax_out, argmax_out, ws, ws_bytes, stream, 1);
}

int bd_masked_ce_workspace_size(int32_t dtype, int32_t n_seqs, int32_t seq_len, int32_t hidden,
                                int32_t vocab, size_t* bytes) {
  if (!bytes || n_seqs <= 0 || seq_len <= 0 || hidden <= 0 || vocab <= 0) return BD_ERR_INVALID_ARG;
  if (dtype != BD_F32 && dtype != BD_BF16) return BD_ERR_UNSUPPORTED;
  if (seq_len % bd::kBlock != 0 || hidden % 8 != 0) return BD_ERR_UNSUPPORTED;
  if (static_cast<long long>(n_seqs) * seq_len > (1LL << 30)) return BD_ERR_INVALID_ARG;
  *bytes = bd::plan_masked_ce(dtype, n_seqs, seq_len, hidden, vocab).total;
  return BD_OK;
}

int bd_masked_ce(int32_t dtype, int32_t n_seqs, int32_t seq_len, int32_t hidden, int32_t vocab,
                 const void* h, const void* w, const int32_t* targets,
                 const uint32_t* masked_bits, float* loss_out, float* loss_sum, int32_t* n_scored,
                 void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("bd_masked_ce");
  if (n_seqs <= 0 || seq_len <= 0 || hidden <= 0 || vocab <= 0) return BD_ERR_INVALID_ARG;
  if (dtype != BD_F32 && dtype != BD_BF16) return BD_ERR_UNSUPPORTED;
  if (seq_len % bd::kBlock != 0 || hidden % 8 != 0) return BD_ERR_UNSUPPORTED;
  if (static_cast<long long>(n_seqs) * seq_len > (1LL << 30)) return BD_ERR_INVALID_ARG;
  if (!h || !w || !targets || !masked_bits || !loss_sum) return BD_ERR_INVALID_ARG;
  // rows are copied and W rows read in 16-byte vectors; W is read by TMA
  if ((reinterpret_cast<uintptr_t>(h) | reinterpret_cast<uintptr_t>(w)) % 16 != 0)
    return BD_ERR_INVALID_ARG;
  const bd::CePlan p = bd::plan_masked_ce(dtype, n_seqs, seq_len, hidden, vocab);
  if (!ws || ws_bytes < p.total) return BD_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return BD_ERR_WORKSPACE;
  return cuda_status(bd::launch_masked_ce(dtype, n_seqs, seq_len, hidden, vocab, p, h, w, targets,
                                          masked_bits, loss_out, loss_sum, n_scored, ws,
                                          static_cast<cudaStream_t>(stream)));
}

int bd_block_mask_attn(const bd_attn_shape* sh, const void* q, const void* k, const void* v,
                       void* out, int32_t n_seqs, int32_t L, int32_t block, void* stream) {
  NvtxRange nvtx_range("bd_block_mask_attn");
  int st = check_shape(sh);
  if (st) return st;
  if (!q || !k || !v || !out || n_seqs <= 0 || n_seqs > 65535 || L <= 0 || block <= 0)
    return BD_ERR_INVALID_ARG;
  if (L % block != 0) return BD_ERR_INVALID_ARG;
  if (L % bd::kBlock != 0 || 2LL * L / bd::kBlock > 2147483647LL) return BD_ERR_UNSUPPORTED;
  return cuda_status(bd::launch_block_mask_attn(*sh, q, k, v, out, n_seqs, L, block,
                                                static_cast<cudaStream_t>(stream)));
}

int bd_block_mask_attn_views(const bd_attn_shape* sh, const void* q, const void* k,
                             const void* v, void* out, int32_t n_seqs, int32_t views, int32_t L,
                             int32_t block, void* stream) {
  NvtxRange nvtx_range("bd_block_mask_attn_views");
  int st = check_shape(sh);
  if (st) return st;
  if (!q || !k || !v || !out || n_seqs <= 0 || n_seqs > 65535 || L <= 0 || block <= 0)
    return BD_ERR_INVALID_ARG;
  if (views <= 0 || n_seqs % views != 0) return BD_ERR_INVALID_ARG;
  if (L % block != 0) return BD_ERR_INVALID_ARG;
  if (L % bd::kBlock != 0 || 2LL * L / bd::kBlock > 2147483647LL) return BD_ERR_UNSUPPORTED;
  return cuda_status(bd::launch_block_mask_attn_views(*sh, q, k, v, out, n_seqs, views, L, block,
                                                      static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
