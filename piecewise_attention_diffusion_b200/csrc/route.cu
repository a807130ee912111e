// bsa_route: covariance-aware top-k block selection.
//
// "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers",
// technical summary §2 (covariance-aware routing): the block score combines the
// attention score with the covariance term M_j = ||H_j - H-bar||, so that relevant or
// heterogeneous blocks are computed exactly and smooth ones go to the Taylor tail.
// The pages give no formula for the combination; this library uses
//     score_ij = softmax_j(s * qbar_i . kbar_j) + lambda * M_j / sum_j' M_j'
// (two distributions, so the mix is scale-free), qbar_i the mean query of block i.
//
// One CTA per (head, query block). The query block is read once with 16-byte loads
// (the only HBM stream; kbar and Mnorm are small and L2-resident), the M block scores
// are warp dot products, and the top-k is an exact rank count with ties broken towards
// the smaller index, compacted in ascending order with a ballot scan.
#include "common.cuh"
#include "internal.h"

namespace bsa {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ float block_reduce(float v, float* s_tmp, bool is_max) {
  v = is_max ? warp_max(v) : warp_sum(v);
  const int w = threadIdx.x / 32;
  __syncthreads();
  if (threadIdx.x % 32 == 0) s_tmp[w] = v;
  __syncthreads();
  float r = s_tmp[0];
  for (int i = 1; i < kWarps; ++i) r = is_max ? fmaxf(r, s_tmp[i]) : r + s_tmp[i];
  return r;
}

template <int B, int D>
__global__ void __launch_bounds__(kThreads)
k_route(const __nv_bfloat16* __restrict__ Q, const float* __restrict__ kbar,
        const float* __restrict__ Mnorm, int L, int k_top, float lambda, float scale,
        int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx,
        float* __restrict__ scores) {
  const int M = L / B;
  const int i = blockIdx.x, bh = blockIdx.y;
  extern __shared__ float s_buf[];
  float* s_qbar = s_buf;                 // D
  float* s_score = s_qbar + D;           // M
  float* s_tmp = s_score + M;            // 32
  float* s_part = s_tmp + 32;            // (kThreads / (D/8)) x D partial column sums
  int* s_wcount = reinterpret_cast<int*>(s_part + kThreads / (D / 8) * D);  // kWarps

  // 1. pooled query: column means over the B rows of block i
  constexpr int CPR = D / 8;               // 16-byte chunks per row
  constexpr int RG = kThreads / CPR;       // row groups
  const int cc = threadIdx.x % CPR, rg = threadIdx.x / CPR;
  const __nv_bfloat16* qb = Q + ((size_t)bh * L + (size_t)i * B) * D;
  float part[8] = {};
  for (int r = rg; r < B; r += RG) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(qb + (size_t)r * D) + cc);
    float f[8];
    bf16x8_to_f32(u, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) part[e] += f[e];
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) s_part[rg * D + cc * 8 + e] = part[e];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += kThreads) {
    float s = 0.f;
    for (int g = 0; g < RG; ++g) s += s_part[g * D + c];
    s_qbar[c] = s * (1.0f / B);
  }
  __syncthreads();

  // 2. block scores a_j = scale * qbar . kbar_j
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const float* kb = kbar + (size_t)bh * M * D;
  for (int j = warp; j < M; j += kWarps) {
    float s = 0.f;
#pragma unroll
    for (int c = lane; c < D; c += 32) s += s_qbar[c] * __ldg(kb + (size_t)j * D + c);
    s = warp_sum(s);
    if (lane == 0) s_score[j] = scale * s;
  }
  __syncthreads();

  // 3. softmax over the M blocks, plus the normalised covariance term
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < M; j += kThreads) mx = fmaxf(mx, s_score[j]);
  mx = block_reduce(mx, s_tmp, true);
  float se = 0.f, sm = 0.f;
  const float* mn = Mnorm + (size_t)bh * M;
  for (int j = threadIdx.x; j < M; j += kThreads) {
    se += expf(s_score[j] - mx);
    sm += __ldg(mn + j);
  }
  se = block_reduce(se, s_tmp, false);
  sm = block_reduce(sm, s_tmp, false);
  const float inv_se = 1.0f / se;
  const float cov = sm > 0.f ? lambda / sm : 0.f;
  __syncthreads();
  for (int j = threadIdx.x; j < M; j += kThreads) {
    const float sc = expf(s_score[j] - mx) * inv_se + cov * __ldg(mn + j);
    s_score[j] = sc;
    if (scores) scores[((size_t)bh * M + i) * M + j] = sc;
  }
  __syncthreads();

  // 4. exact top-k by rank count; 5. ascending compaction with a ballot scan
  const int64_t head_base = (int64_t)bh * M * k_top;
  int base = 0;
  for (int j0 = 0; j0 < M; j0 += kThreads) {
    const int j = j0 + threadIdx.x;
    bool sel = false;
    if (j < M) {
      const float sj = s_score[j];
      int rank = 0;
      for (int jj = 0; jj < M; ++jj) {
        const float o = s_score[jj];
        rank += (o > sj || (o == sj && jj < j)) ? 1 : 0;
      }
      sel = rank < k_top;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, sel);
    if (lane == 0) s_wcount[warp] = __popc(bal);
    __syncthreads();
    int pos = base + __popc(bal & ((1u << lane) - 1u));
    for (int w = 0; w < warp; ++w) pos += s_wcount[w];
    if (sel) col_idx[head_base + (int64_t)i * k_top + pos] = j;
    int tot = 0;
    for (int w = 0; w < kWarps; ++w) tot += s_wcount[w];
    base += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    int32_t* rp = row_ptr + (size_t)bh * (M + 1);
    rp[i] = (int32_t)(head_base + (int64_t)i * k_top);
    if (i == M - 1) rp[M] = (int32_t)(head_base + (int64_t)M * k_top);
  }
}

template <int B, int D>
cudaError_t run(const Shape& s, const void* Q, const float* kbar, const float* Mnorm,
                int k_top, float lambda, float scale, int32_t* row_ptr, int32_t* col_idx,
                float* scores, cudaStream_t st) {
  const int M = s.M();
  const size_t sm = (D + M + 32 + (size_t)kThreads / (D / 8) * D) * sizeof(float) +
                    kWarps * sizeof(int);
  cudaError_t e = cudaFuncSetAttribute(k_route<B, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  k_route<B, D><<<dim3(M, s.BH()), kThreads, sm, st>>>(
      static_cast<const __nv_bfloat16*>(Q), kbar, Mnorm, s.L, k_top, lambda, scale, row_ptr,
      col_idx, scores);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const Shape& s, const void* Q, const float* kbar, const float* Mnorm,
                         int k_top, float lambda, float scale, int32_t* row_ptr,
                         int32_t* col_idx, float* scores, int32_t* status, cudaStream_t st) {
  (void)status;
  if (s.block == 64 && s.d == 64)
    return run<64, 64>(s, Q, kbar, Mnorm, k_top, lambda, scale, row_ptr, col_idx, scores, st);
  if (s.block == 64 && s.d == 128)
    return run<64, 128>(s, Q, kbar, Mnorm, k_top, lambda, scale, row_ptr, col_idx, scores, st);
  if (s.block == 128 && s.d == 64)
    return run<128, 64>(s, Q, kbar, Mnorm, k_top, lambda, scale, row_ptr, col_idx, scores, st);
  return run<128, 128>(s, Q, kbar, Mnorm, k_top, lambda, scale, row_ptr, col_idx, scores, st);
}

}  // namespace bsa
