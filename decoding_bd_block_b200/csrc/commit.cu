// bd_cache_commit: rotate the keys of finished blocks at their absolute
// positions and append K/V as pages of the block-level KV cache
// ("Fast-dLLM v2: Efficient Block-Diffusion LLM", key design 3: a decoded
// block becomes read-only context for later blocks).
#include "bd_common.cuh"

namespace bd {
namespace {

// grid (32 * n_new_blocks, n_seqs); one CTA per committed token.
template <typename T>
__global__ void __launch_bounds__(128) cache_commit_kernel(
    T* __restrict__ pages, long long n_pages, const int32_t* __restrict__ page_table,
    int max_blocks, int32_t* __restrict__ n_blocks, const T* __restrict__ k,
    const T* __restrict__ v, int Hkv, int d, double theta, CommitArgs a) {
  __shared__ float cs[64];
  __shared__ float sn[64];
  const int t = blockIdx.x;
  const int si = blockIdx.y;
  const int s = a.seq_ids[si];
  const int first = a.first_block[si];
  const int half = d / 2;
  const long long pos = static_cast<long long>(first) * kBlock + t;
  for (int j = threadIdx.x; j < half; j += blockDim.x)
    rope_cos_sin(pos, rope_inv_freq(j, d, theta), &cs[j], &sn[j]);
  __syncthreads();

  if (t == 0 && threadIdx.x == 0) n_blocks[s] = first + a.n_new_blocks;
  const int page = page_table[static_cast<size_t>(s) * max_blocks + first + t / kBlock];
  BD_CHECK(page >= 0 && page < n_pages, kCheckPageId, page);
  if (page < 0 || page >= n_pages) return;  // host-validated; never write outside the pool
  const int row = t % kBlock;
  const size_t span = static_cast<size_t>(kBlock) * a.n_new_blocks;
  const T* ks = k + (static_cast<size_t>(si) * span + t) * Hkv * d;
  const T* vs = v + (static_cast<size_t>(si) * span + t) * Hkv * d;
  for (int idx = threadIdx.x; idx < Hkv * half; idx += blockDim.x) {
    const int g = idx / half, j = idx % half;
    const float x1 = to_f32(ks[g * d + j]);
    const float x2 = to_f32(ks[g * d + j + half]);
    T* kd = pages + ((static_cast<size_t>(page) * 2 + 0) * Hkv + g) * kBlock * d + row * d;
    kd[j] = from_f32<T>(x1 * cs[j] - x2 * sn[j]);
    kd[j + half] = from_f32<T>(x2 * cs[j] + x1 * sn[j]);
  }
  for (int idx = threadIdx.x; idx < Hkv * d; idx += blockDim.x) {
    const int g = idx / d, c = idx % d;
    pages[((static_cast<size_t>(page) * 2 + 1) * Hkv + g) * kBlock * d + row * d + c] = vs[g * d + c];
  }
}

}  // namespace

cudaError_t launch_cache_commit(const bd_attn_shape& sh, const bd_kv_cache& c, const void* k,
                                const void* v, const CommitArgs& a, cudaStream_t st) {
  dim3 grid(kBlock * a.n_new_blocks, a.n_seqs);
  if (sh.dtype == BD_BF16)
    cache_commit_kernel<bf16><<<grid, 128, 0, st>>>(
        static_cast<bf16*>(c.pages), c.n_pages, c.page_table, c.max_blocks, c.n_blocks,
        static_cast<const bf16*>(k), static_cast<const bf16*>(v), sh.n_heads_kv, sh.head_dim,
        sh.rope_theta, a);
  else
    cache_commit_kernel<float><<<grid, 128, 0, st>>>(
        static_cast<float*>(c.pages), c.n_pages, c.page_table, c.max_blocks, c.n_blocks,
        static_cast<const float*>(k), static_cast<const float*>(v), sh.n_heads_kv, sh.head_dim,
        sh.rope_theta, a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace bd

#ifdef BD_DEVICE_CHECKS
namespace bd {
cudaError_t check_word_commit(int* host2, bool reset) { return read_check_word(host2, reset); }
}  // namespace bd
#endif
