// bsa_forward: fused online-softmax attention over block lists, keep-or-drop or PISA.
//
// "多模态 DiT 上的块稀疏 Attention" §3.3/§4.3/§4.4: per query block i, softmax over the
// selected key blocks S_i only, computed with an online softmax inside each block pair.
// "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers",
// technical summary §2: blocks outside S_i enter the same numerator and denominator
// through alpha_tj = exp(s q_t . kbar_j) (zeroth order, value sum vsum_j, weight B in
// the denominator) and one global first-order term s (q_t Hbar) sum_{U_i} alpha_tj.
//
// This file holds the launch sequence: a validation pass over the block lists (a
// malformed list sets BSA_ERR_BAD_CSR and the attention kernel leaves O untouched; with
// token padding, a real-token count outside 1..block or, in the PISA modes, a list that
// lacks a padded block sets BSA_ERR_BAD_PADDING the same way), then the tensor-core
// attention kernel (forward_tc.cu dispatches by mode and head dim: forward_tc.cu for
// head dim 128 and the per-block mode, forward_pair.cu for head dim 64).
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace bsa {
namespace {

// One warp per row: the lanes read the row's entries 32 at a time (coalesced), each
// entry is compared with its left neighbour (the previous chunk's last entry carried in
// lane 0), and the PISA count of padded blocks in the row is a warp sum.
__global__ void k_validate_csr(const int32_t* __restrict__ row_ptr,
                               const int32_t* __restrict__ col_idx, int64_t nnz_total, int M,
                               int n_heads, const int32_t* __restrict__ key_valid, int block,
                               bool pisa, int32_t* flag, int32_t* status) {
  constexpr int kWarps = 8;
  __shared__ int s_npad;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_rows = n_heads * M;
  // padded blocks (real tokens < block) and the range of every count
  if (threadIdx.x == 0) s_npad = 0;
  __syncthreads();
  if (key_valid != nullptr) {
    int mine = 0;
    for (int j = threadIdx.x; j < M; j += blockDim.x) {
      const int v = __ldg(key_valid + j);
      mine += v < block ? 1 : 0;
      if ((v < 1 || v > block) && blockIdx.x == 0) {
        atomicOr(flag, 1);
        report(status, BSA_ERR_BAD_PADDING);
      }
    }
    mine = __reduce_add_sync(0xffffffffu, mine);
    if (lane == 0 && mine) atomicAdd(&s_npad, mine);
  }
  __syncthreads();
  const int n_pad = s_npad;
  for (int r = blockIdx.x * kWarps + warp; r < n_rows; r += gridDim.x * kWarps) {
    const int h = r / M, i = r % M;
    const int32_t* rp = row_ptr + (size_t)h * (M + 1);
    const int64_t b = __ldg(rp + i), e = __ldg(rp + i + 1);
    bool ok = b >= 0 && b <= e && e <= nnz_total && (e - b) <= M;
    int prev = -1, in_row = 0;
    if (ok) {
      for (int64_t p0 = b; p0 < e; p0 += 32) {
        const int64_t p = p0 + lane;
        const bool has = p < e;
        const int c = has ? __ldg(col_idx + p) : 0;
        int left = __shfl_up_sync(0xffffffffu, c, 1);
        if (lane == 0) left = prev;
        if (__any_sync(0xffffffffu, has && (c <= left || c >= M))) {
          ok = false;
          break;
        }
        const int64_t rem = e - 1 - p0;
        const int last = rem < 31 ? (int)rem : 31;
        prev = __shfl_sync(0xffffffffu, c, last);
        if (pisa && n_pad > 0 && has) in_row += __ldg(key_valid + c) < block ? 1 : 0;
      }
    }
    if (!ok) {
      if (lane == 0) {
        atomicOr(flag, 1);
        report(status, BSA_ERR_BAD_CSR);
      }
    } else if (pisa && n_pad > 0) {
      // a padded block is always computed exactly: it must be in every list
      in_row = __reduce_add_sync(0xffffffffu, in_row);
      if (in_row != n_pad && lane == 0) {
        atomicOr(flag, 1);
        report(status, BSA_ERR_BAD_PADDING);
      }
    }
  }
}

}  // namespace

size_t forward_workspace(const Shape& s) { return forward_tc_workspace(s); }

cudaError_t launch_forward(const ForwardArgs& args, cudaStream_t st) {
  ForwardArgs a = args;
  a.scale = forward_scale(args.scale, args.s.d);
  const Shape& s = a.s;
  const int M = s.M();
  int32_t* flag = static_cast<int32_t*>(a.ws);
  cudaError_t e = cudaMemsetAsync(flag, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return e;
  const int n_heads = a.csr_per_head ? s.BH() : 1;
  const int rows = n_heads * M;
  k_validate_csr<<<ceil_div(rows, 8), 256, 0, st>>>(
      a.row_ptr, a.col_idx, a.nnz_total, M, n_heads, s.key_valid, s.block,
      a.mode == BSA_MODE_PISA || a.mode == BSA_MODE_PISA_BLOCK, flag, a.status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_forward_tc(a, flag, st);
}

}  // namespace bsa
