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
// malformed list sets BSA_ERR_BAD_CSR and the attention kernel leaves O untouched),
// then the attention kernel. The attention kernel here is a straightforward one-warp-
// per-query-row formulation on the CUDA cores.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace bsa {
namespace {

// Workspace layout: [0, 256) validation flag.
constexpr size_t kFlagBytes = 256;

__global__ void k_validate_csr(const int32_t* __restrict__ row_ptr,
                               const int32_t* __restrict__ col_idx, int64_t nnz_total, int M,
                               int n_heads, int32_t* flag, int32_t* status) {
  const int n_rows = n_heads * M;
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
    }
  }
}

template <int D>
__global__ void __launch_bounds__(128)
k_fwd_rowwise(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
              const __nv_bfloat16* __restrict__ V, int L, int B,
              const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
              int csr_per_head, int mode, const float* __restrict__ kbar,
              const float* __restrict__ vsum, const float* __restrict__ Hbar, float scale,
              __nv_bfloat16* __restrict__ O, float* __restrict__ lse,
              const int32_t* __restrict__ flag) {
  if (*flag) return;
  constexpr int E = D / 32;  // elements per lane (lane + 32 e)
  const int lane = threadIdx.x % 32;
  const int t = blockIdx.x * 4 + threadIdx.x / 32;
  const int bh = blockIdx.y;
  if (t >= L) return;
  const int M = L / B, i = t / B;
  const int32_t* rp = csr_per_head ? row_ptr + (size_t)bh * (M + 1) : row_ptr;
  const int beg = rp[i], end = rp[i + 1];
  const size_t head = (size_t)bh * L * D;

  float q[E], o[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    q[e] = __bfloat162float(Q[head + (size_t)t * D + lane + 32 * e]);
    o[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f, sa = 0.f;

  // exact terms over S_i
  for (int p = beg; p < end; ++p) {
    const int j = col_idx[p];
    for (int n = 0; n < B; ++n) {
      const size_t key = head + ((size_t)j * B + n) * D;
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) s += q[e] * __bfloat162float(K[key + lane + 32 * e]);
      s = scale * warp_sum(s);
      const float mn = fmaxf(m, s);
      const float c = expf(m - mn), pe = expf(s - mn);
      l = l * c + pe;
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = o[e] * c + pe * __bfloat162float(V[key + lane + 32 * e]);
      m = mn;
    }
  }

  if (mode == BSA_MODE_PISA) {
    // zeroth-order centroid terms over U_i = complement of the (ascending) list
    const float* kb = kbar + (size_t)bh * M * D;
    const float* vs = vsum + (size_t)bh * M * D;
    int p = beg;
    for (int j = 0; j < M; ++j) {
      if (p < end && col_idx[p] == j) {
        ++p;
        continue;
      }
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) a += q[e] * kb[(size_t)j * D + lane + 32 * e];
      a = scale * warp_sum(a);
      const float mn = fmaxf(m, a);
      const float c = expf(m - mn), al = expf(a - mn);
      l = l * c + (float)B * al;
      sa = sa * c + al;
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = o[e] * c + al * vs[(size_t)j * D + lane + 32 * e];
      m = mn;
    }
    // global first-order correction: s * (q Hbar) * sum alpha
    const float* hb = Hbar + (size_t)bh * D * D;
    float qh[E] = {};
#pragma unroll
    for (int ea = 0; ea < E; ++ea)
      for (int src = 0; src < 32; ++src) {
        const float qa = __shfl_sync(0xffffffffu, q[ea], src);
        const int a = src + 32 * ea;
#pragma unroll
        for (int e = 0; e < E; ++e) qh[e] += qa * hb[(size_t)a * D + lane + 32 * e];
      }
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] += scale * sa * qh[e];
  }

  const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) O[head + (size_t)t * D + lane + 32 * e] = __float2bfloat16(o[e] * inv);
  if (lse && lane == 0) lse[(size_t)bh * L + t] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace

size_t forward_workspace(const Shape& s) {
  (void)s;
  return kFlagBytes;
}

cudaError_t launch_forward(const ForwardArgs& a, cudaStream_t st) {
  const Shape& s = a.s;
  const int M = s.M();
  int32_t* flag = static_cast<int32_t*>(a.ws);
  cudaError_t e = cudaMemsetAsync(flag, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return e;
  const int n_heads = a.csr_per_head ? s.BH() : 1;
  const int rows = n_heads * M;
  k_validate_csr<<<ceil_div(rows, 256), 256, 0, st>>>(a.row_ptr, a.col_idx, a.nnz_total, M,
                                                      n_heads, flag, a.status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const dim3 grid(ceil_div(s.L, 4), s.BH());
  const auto* Qb = static_cast<const __nv_bfloat16*>(a.Q);
  const auto* Kb = static_cast<const __nv_bfloat16*>(a.K);
  const auto* Vb = static_cast<const __nv_bfloat16*>(a.V);
  auto* Ob = static_cast<__nv_bfloat16*>(a.O);
  if (s.d == 64)
    k_fwd_rowwise<64><<<grid, 128, 0, st>>>(Qb, Kb, Vb, s.L, s.block, a.row_ptr, a.col_idx,
                                            a.csr_per_head, a.mode, a.kbar, a.vsum, a.Hbar,
                                            a.scale, Ob, a.lse, flag);
  else
    k_fwd_rowwise<128><<<grid, 128, 0, st>>>(Qb, Kb, Vb, s.L, s.block, a.row_ptr, a.col_idx,
                                             a.csr_per_head, a.mode, a.kbar, a.vsum, a.Hbar,
                                             a.scale, Ob, a.lse, flag);
  return cudaGetLastError();
}

}  // namespace bsa
