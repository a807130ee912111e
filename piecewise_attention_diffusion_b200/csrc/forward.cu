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
// attention kernel of forward_tc.cu.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace bsa {
namespace {

__global__ void k_validate_csr(const int32_t* __restrict__ row_ptr,
                               const int32_t* __restrict__ col_idx, int64_t nnz_total, int M,
                               int n_heads, const int32_t* __restrict__ key_valid, int block,
                               bool pisa, int32_t* flag, int32_t* status) {
  const int n_rows = n_heads * M;
  // padded blocks (real tokens < block) and the range of every count
  int n_pad = 0;
  if (key_valid != nullptr) {
    for (int j = 0; j < M; ++j) {
      const int v = __ldg(key_valid + j);
      n_pad += v < block ? 1 : 0;
      if ((v < 1 || v > block) && blockIdx.x == 0 && threadIdx.x == 0) {
        atomicOr(flag, 1);
        report(status, BSA_ERR_BAD_PADDING);
      }
    }
  }
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < n_rows; r += gridDim.x * blockDim.x) {
    const int h = r / M, i = r % M;
    const int32_t* rp = row_ptr + (size_t)h * (M + 1);
    const int64_t b = rp[i], e = rp[i + 1];
    bool ok = b >= 0 && b <= e && e <= nnz_total && (e - b) <= M;
    if (ok) {
      int prev = -1;
      for (int64_t p = b; p < e; ++p) {
        const int c = col_idx[p];
        if (c <= prev || c >= M) {
          ok = false;
          break;
        }
        prev = c;
      }
    }
    if (!ok) {
      atomicOr(flag, 1);
      report(status, BSA_ERR_BAD_CSR);
    } else if (pisa && n_pad > 0) {
      // a padded block is always computed exactly: it must be in every list
      int in_row = 0;
      for (int64_t p = b; p < e; ++p) in_row += __ldg(key_valid + col_idx[p]) < block ? 1 : 0;
      if (in_row != n_pad) {
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
  k_validate_csr<<<ceil_div(rows, 256), 256, 0, st>>>(
      a.row_ptr, a.col_idx, a.nnz_total, M, n_heads, s.key_valid, s.block,
      a.mode == BSA_MODE_PISA || a.mode == BSA_MODE_PISA_BLOCK, flag, a.status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_forward_tc(a, flag, st);
}

}  // namespace bsa
