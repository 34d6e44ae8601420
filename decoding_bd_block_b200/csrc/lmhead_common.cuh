// Pieces shared by the two tensor-core LM-head kernels (select_tc.cu: packed
// rows streamed by TMA; select_fused.cu: rows resident in shared memory):
// tile constants, the per-chunk fold of logits into (max, sum, argmax), and
// the 2-D bf16 tensor maps that stream W.
#pragma once

#include <cuda.h>

#include "bd_common.cuh"
#include "tc_common.cuh"

namespace bd {
namespace lmh {

constexpr int kVTile = 128;                    // vocab rows per MMA (M)
constexpr int kKStage = 64;                    // hidden elements per K-slice (128 B rows)
constexpr int kWBytes = kVTile * kKStage * 2;  // 16 KB: one W slice of a tile

__device__ __forceinline__ int round16(int x) { return (x + 15) & ~15; }

// Running (max, sum exp, argmax) of one packed row's logits.
struct Run {
  float m, s;
  int a;
};
__device__ __forceinline__ Run run_empty() { return Run{-INFINITY, 0.f, 0x7fffffff}; }

// Folds one 32 x 32 chunk of the accumulator -- TMEM lanes = 32 vocab rows
// starting at vocab row `vbase`, columns = 32 packed rows -- into the
// running statistics of column `lane`, kept by that lane.  The chunk goes
// through the warp's 32 x 33 buffer `tb` transposed, so each thread then
// folds one column with plain per-thread arithmetic.  Vocab rows >= vend are
// outside the tile and skipped.  Ties keep the lowest vocab index.
__device__ __forceinline__ void fold_chunk(uint32_t taddr, float* tb, int lane, int vbase,
                                           int vend, Run& run) {
  uint32_t r[32];
  tc::tmem_ld_32x32b_x32(taddr, r);
  tc::tmem_ld_wait();
#pragma unroll
  for (int j = 0; j < 32; ++j) tb[j * 33 + lane] = __uint_as_float(r[j]);
  __syncwarp();
  const bool full = vbase + 32 <= vend;
  const float* col = tb + lane * 33;
  float mk[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  int ak[4] = {0, 0, 0, 0};
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float x = (full || vbase + i < vend) ? col[i] : -INFINITY;
    if (x > mk[i & 3]) {
      mk[i & 3] = x;
      ak[i & 3] = i;
    }
  }
  const float mx = fmaxf(fmaxf(mk[0], mk[1]), fmaxf(mk[2], mk[3]));
  int am = 32;
#pragma unroll
  for (int k = 0; k < 4; ++k) am = (mk[k] == mx && ak[k] < am) ? ak[k] : am;
  if (mx != -INFINITY) {
    const float mls = mx * kLog2e;
    float sk[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float x = (full || vbase + i < vend) ? col[i] : -INFINITY;
      sk[i & 3] += fast_exp2(fmaf(x, kLog2e, -mls));
    }
    const float e = (sk[0] + sk[1]) + (sk[2] + sk[3]);
    const int arg = vbase + am;
    if (mx > run.m) {
      run.s = run.s * fast_exp2((run.m - mx) * kLog2e) + e;
      run.m = mx;
      run.a = arg;
    } else {
      run.s += e * fast_exp2((mx - run.m) * kLog2e);
      if (mx == run.m && arg < run.a) run.a = arg;
    }
  }
  __syncwarp();
}

// ------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 tensor [rows][cols] (row-major), tile box [box_rows][64 cols],
// 128-byte swizzle, zero fill outside the tensor.
inline bool make_tmap_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                         uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline int sm_count() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

}  // namespace lmh
}  // namespace bd
