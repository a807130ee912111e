// bsa_build_mask: the multimodal fixed block pattern as CSR index lists.
//
// "多模态 DiT 上的块稀疏 Attention" §4.2 builds a dense 0/1 block matrix: text rows and
// text columns full; image-to-image kept inside a local window or on a global column
// every `global_stride` blocks. §5.4 recommends per-query-block index lists instead of
// the dense matrix, and §8.1 builds them once and reuses them. Here the window is the
// Chebyshev neighbourhood on a 2-D grid of image blocks (grid_h = 1 gives the page's
// 1-D |i - j| <= window). One CTA: M is at most a few thousand blocks and the pattern
// is built once per model, so the kernel is launch-bound by design.
#include "common.cuh"
#include "internal.h"

namespace bsa {
namespace {

__device__ __forceinline__ bool keeps(const bsa_mask_desc& d, int i, int j) {
  const int nt = d.n_text_blocks;
  if (i < nt || j < nt) return true;
  const int a = i - nt, b = j - nt;
  const int dr = abs(a / d.grid_w - b / d.grid_w);
  const int dc = abs(a % d.grid_w - b % d.grid_w);
  if (max(dr, dc) <= d.radius) return true;
  if (d.global_stride > 0) {
    if (b % d.global_stride == 0) return true;
    if (d.global_rows_full && a % d.global_stride == 0) return true;
  }
  return false;
}

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
k_build_mask(bsa_mask_desc desc, int M, int32_t* row_ptr, int32_t* col_idx, int64_t cap,
             int32_t* status) {
  extern __shared__ int32_t s_len[];  // M + 1 entries
  for (int i = threadIdx.x; i < M; i += blockDim.x) {
    int n = 0;
    for (int j = 0; j < M; ++j) n += keeps(desc, i, j) ? 1 : 0;
    s_len[i] = n;
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // exclusive scan; M <= 2048 so a serial pass is cheap
    int acc = 0;
    for (int i = 0; i < M; ++i) {
      const int n = s_len[i];
      s_len[i] = acc;
      acc += n;
    }
    s_len[M] = acc;
  }
  __syncthreads();
  for (int i = threadIdx.x; i <= M; i += blockDim.x) row_ptr[i] = s_len[i];
  if ((int64_t)s_len[M] > cap) {
    if (threadIdx.x == 0) report(status, BSA_ERR_CAPACITY);
    return;
  }
  for (int i = threadIdx.x; i < M; i += blockDim.x) {
    int p = s_len[i];
    for (int j = 0; j < M; ++j)
      if (keeps(desc, i, j)) col_idx[p++] = j;
  }
}

}  // namespace

cudaError_t launch_build_mask(const bsa_mask_desc& desc, int M, int32_t* row_ptr,
                              int32_t* col_idx, int64_t cap, int32_t* status,
                              cudaStream_t st) {
  k_build_mask<<<1, kThreads, (M + 1) * sizeof(int32_t), st>>>(desc, M, row_ptr, col_idx,
                                                               cap, status);
  return cudaGetLastError();
}

}  // namespace bsa
