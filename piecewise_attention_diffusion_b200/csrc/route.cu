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
// One CTA per (head, 8 query blocks), one warp per query block:
//   1. pooled query: the warp streams its block of Q with 16-byte loads (the only HBM
//      stream of the call) and reduces the columns;
//   2. scores: thread t takes centroid j = t (looping when M > 256; with M <= 128 two
//      threads share a centroid, half of d each, and add across the pair), reads its row
//      once per CTA (16-byte loads from L2) and dots it with the CTA's 8 pooled queries,
//      which every thread reads from the same shared-memory words (broadcast);
//   3. softmax over the M blocks plus the normalised covariance term;
//   4. exact top-k: the k-th largest score is found by a radix select on the float bit
//      patterns (scores are >= 0, so the bit patterns order like the values), ties at
//      the threshold go to the smaller block index, and the selected indices are
//      compacted in ascending order with ordered ballots.
// Token padding: the pooled query of a block averages its real rows only, and every
// padded block (fewer than B real tokens) is forced into every list. It takes the key
// +inf in the selection (scores are finite), so the radix select, the tie rule and the
// compaction treat it as the largest score without a separate pass; the scores
// written out keep the real values.
#include "common.cuh"
#include "internal.h"

namespace bsa {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr uint32_t kForcedKey = 0x7F800000u;  // bit pattern of +inf

template <int B, int D>
__global__ void __launch_bounds__(kThreads)
k_route(const __nv_bfloat16* __restrict__ Q, const float* __restrict__ kbar,
        const float* __restrict__ Mnorm, const int32_t* __restrict__ key_valid, int L,
        int k_top, float lambda, float scale, int32_t* __restrict__ row_ptr,
        int32_t* __restrict__ col_idx, float* __restrict__ scores, int32_t* status) {
  const int M = L / B;
  const int bh = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int i = blockIdx.x * kWarps + warp;  // this warp's query block
  const bool active = i < M;

  extern __shared__ __align__(16) float smem[];
  float* s_q = smem;                            // kWarps x D (16-byte aligned rows)
  float* s_cov = s_q + kWarps * D;              // M
  float* s_sc = s_cov + M;                      // kWarps x M
  float* s_red = s_sc + kWarps * M;             // kWarps

  // normalised covariance term, shared by every query block of the head
  const float* mn = Mnorm + (size_t)bh * M;
  float part = 0.f;
  for (int j = threadIdx.x; j < M; j += kThreads) part += __ldg(mn + j);
  part = warp_sum(part);
  if (lane == 0) s_red[warp] = part;
  __syncthreads();
  float msum = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) msum += s_red[w];
  const float cov = msum > 0.f ? lambda / msum : 0.f;
  for (int j = threadIdx.x; j < M; j += kThreads) s_cov[j] = cov * __ldg(mn + j);

  // 1. pooled query of block i: lanes 0..CPR-1 take row r, the next CPR lanes row r+1...
  constexpr int CPR = D / 8;          // 16-byte chunks per row
  constexpr int RPI = 32 / CPR;       // rows per warp iteration
  constexpr int kUnrollQ = B / RPI >= 32 ? 16 : 8;  // loads in flight per lane
  float* qbar = s_q + warp * D;
  if (active) {
    const __nv_bfloat16* qb = Q + ((size_t)bh * L + (size_t)i * B) * D;
    const int cc = lane % CPR, r0 = lane / CPR;
    int nq = B;  // real query rows of block i
    if (key_valid != nullptr) {
      const int raw = __ldg(key_valid + i);
      if ((raw < 1 || raw > B) && lane == 0) report(status, BSA_ERR_BAD_PADDING);
      nq = min(max(raw, 1), B);
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll kUnrollQ
    for (int r = r0; r < B; r += RPI) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(qb + (size_t)r * D) + cc);
      float f[8];
      bf16x8_to_f32(u, f);
      if (r < nq) {
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += f[e];
      }
    }
#pragma unroll
    for (int o = CPR; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    if (lane < CPR) {
#pragma unroll
      for (int e = 0; e < 8; ++e) qbar[cc * 8 + e] = acc[e] / (float)nq;
    }
  }
  __syncwarp();

  // 2. block scores a_j = scale * qbar_w . kbar_j for the CTA's query blocks
  const float* kb = kbar + (size_t)bh * M * D;
  float* sc = s_sc + warp * M;
  if (!active) {
#pragma unroll 1
    for (int c = lane; c < D; c += 32) qbar[c] = 0.f;  // keep the dots below finite
  }
  __syncthreads();
  // 16-byte loads when the caller's kbar allows them (each head's slice then does too,
  // since M * D * 4 is a multiple of 16)
  const bool vec = (reinterpret_cast<uintptr_t>(kbar) & 15u) == 0;
  // with at most kThreads / 2 centroids two threads share one (half of d each)
  const int split = 2 * M <= kThreads ? 2 : 1;
  const int total = M * split;
  for (int base = warp * 32; base < total; base += kThreads) {
    const int jj = base + lane;
    const bool valid = jj < total;
    const int j = valid ? jj / split : 0, part = jj % split;
    float acc[kWarps];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) acc[w] = 0.f;
    const float* kr = kb + (size_t)j * D;
    const int cb = part * (D / split), ce = cb + D / split;
#pragma unroll 4
    for (int c = cb; c < ce; c += 4) {
      float4 kv;
      if (vec) {
        kv = __ldg(reinterpret_cast<const float4*>(kr + c));
      } else {
        kv = make_float4(__ldg(kr + c), __ldg(kr + c + 1), __ldg(kr + c + 2), __ldg(kr + c + 3));
      }
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float4 qv = *reinterpret_cast<const float4*>(s_q + w * D + c);
        acc[w] = fmaf(qv.w, kv.w, fmaf(qv.z, kv.z, fmaf(qv.y, kv.y, fmaf(qv.x, kv.x, acc[w]))));
      }
    }
    if (split == 2) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) acc[w] += __shfl_xor_sync(0xffffffffu, acc[w], 1);
    }
    if (valid && part == 0) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s_sc[w * M + j] = scale * acc[w];
    }
  }
  __syncthreads();
  __syncwarp();
  if (!active) return;

  // 3. softmax over the M blocks plus the covariance term
  float mx = -INFINITY;
  for (int j = lane; j < M; j += 32) mx = fmaxf(mx, sc[j]);
  mx = warp_max(mx);
  float se = 0.f;
  for (int j = lane; j < M; j += 32) se += expf(sc[j] - mx);
  se = warp_sum(se);
  const float inv_se = 1.0f / se;
  float* srow = scores ? scores + ((size_t)bh * M + i) * M : nullptr;
  int n_forced = 0;
  for (int j = lane; j < M; j += 32) {
    const float v = expf(sc[j] - mx) * inv_se + s_cov[j];
    const bool forced = key_valid != nullptr && __ldg(key_valid + j) < B;
    n_forced += forced ? 1 : 0;
    sc[j] = forced ? __uint_as_float(kForcedKey) : v;
    if (srow) srow[j] = v;
  }
  n_forced = __reduce_add_sync(0xffffffffu, n_forced);
  if (n_forced > k_top) {
    // the list cannot hold every padded block: report, and emit a valid list anyway
    if (lane == 0) report(status, BSA_ERR_BAD_PADDING);
    for (int j = lane; j < M; j += 32)
      if (__float_as_uint(sc[j]) == kForcedKey) sc[j] = 0.f;
  }
  __syncwarp();

  // 4. k-th largest key (bit pattern of a non-negative float) by radix select
  uint32_t T = 0;
  if (M <= 128) {
    // up to 4 keys per lane, held in registers for the 32 passes (absent keys 0: never
    // counted, every candidate has a bit set)
    uint32_t key[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = lane + 32 * q;
      key[q] = j < M ? __float_as_uint(sc[j]) : 0u;
    }
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      int cnt = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) cnt += key[q] >= cand ? 1 : 0;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (cnt >= k_top) T = cand;
    }
  } else {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      int cnt = 0;
      for (int j = lane; j < M; j += 32) cnt += __float_as_uint(sc[j]) >= cand ? 1 : 0;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (cnt >= k_top) T = cand;
    }
  }
  int greater = 0;
  for (int j = lane; j < M; j += 32) greater += __float_as_uint(sc[j]) > T ? 1 : 0;
  greater = __reduce_add_sync(0xffffffffu, greater);
  const int ties_needed = k_top - greater;  // >= 1

  // 5. ascending compaction: selected = key > T, or key == T among the first
  //    ties_needed such keys in index order
  const int64_t base = (int64_t)bh * M * k_top + (int64_t)i * k_top;
  const unsigned lt = (1u << lane) - 1u;
  int ties_seen = 0, out = 0;
  for (int j0 = 0; j0 < M; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < M ? __float_as_uint(sc[j]) : 0u;
    const bool tie = j < M && key == T;
    const unsigned tb = __ballot_sync(0xffffffffu, tie);
    const bool sel = j < M && (key > T || (tie && ties_seen + __popc(tb & lt) < ties_needed));
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    if (sel) col_idx[base + out + __popc(sb & lt)] = j;
    ties_seen += __popc(tb);
    out += __popc(sb);
  }
  if (lane == 0) {
    int32_t* rp = row_ptr + (size_t)bh * (M + 1);
    rp[i] = (int32_t)base;
    if (i == M - 1) rp[M] = (int32_t)((int64_t)bh * M * k_top + (int64_t)M * k_top);
  }
}

template <int B, int D>
cudaError_t run(const Shape& s, const void* Q, const float* kbar, const float* Mnorm,
                int k_top, float lambda, float scale, int32_t* row_ptr, int32_t* col_idx,
                float* scores, int32_t* status, cudaStream_t st) {
  const int M = s.M();
  const size_t sm = ((size_t)kWarps * D + M + (size_t)kWarps * M + kWarps) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(k_route<B, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  k_route<B, D><<<dim3(ceil_div(M, kWarps), s.BH()), kThreads, sm, st>>>(
      static_cast<const __nv_bfloat16*>(Q), kbar, Mnorm, s.key_valid, s.L, k_top, lambda, scale,
      row_ptr, col_idx, scores, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const Shape& s, const void* Q, const float* kbar, const float* Mnorm,
                         int k_top, float lambda, float scale, int32_t* row_ptr,
                         int32_t* col_idx, float* scores, int32_t* status, cudaStream_t st) {
  if (s.block == 64 && s.d == 64)
    return run<64, 64>(s, Q, kbar, Mnorm, k_top, lambda, scale, row_ptr, col_idx, scores,
                        status, st);
  if (s.block == 64 && s.d == 128)
    return run<64, 128>(s, Q, kbar, Mnorm, k_top, lambda, scale, row_ptr, col_idx, scores,
                         status, st);
  if (s.block == 128 && s.d == 64)
    return run<128, 64>(s, Q, kbar, Mnorm, k_top, lambda, scale, row_ptr, col_idx, scores,
                         status, st);
  return run<128, 128>(s, Q, kbar, Mnorm, k_top, lambda, scale, row_ptr, col_idx, scores,
                          status, st);
}

}  // namespace bsa
