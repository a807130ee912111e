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
// Two kernels:
//   k_pool   streams Q once (the only large read of the call): one warp sums a segment
//            of 32 rows with 16-byte loads, all of them in flight at once, and writes the
//            column sums to the workspace (one slot per segment; no atomics, so the sums
//            are the same bits on every run). Segments are dealt to a grid of a few CTAs
//            per SM in a loop, so no SM is left with a partial last wave of long work;
//   k_route  one CTA per (head, 8 query blocks), one warp per query block:
//     1. pooled query: the sum of the block's segment sums (workspace, L2) over its
//        number of real rows;
//     2. scores: eight lanes share a centroid row, so that every copy of kbar (from L2)
//        reads whole 128-byte segments, and dot it with the CTA's 8 pooled queries in
//        shared memory; each lane takes two rows, so that every pooled-query chunk it
//        reads serves both; a butterfly over the eight lanes adds the partial dots. Each
//        lane copies (cp.async) its chunks of the next pass's rows into its own slots of
//        shared memory while it computes this pass;
//     3. softmax over the M blocks plus the normalised covariance term;
//     4. exact top-k: a threshold of the k largest scores is found by a radix select on
//        the float bit patterns (scores are >= 0, so the bit patterns order like the
//        values), bit by bit until exactly k keys are at or above it, or to the last bit,
//        with the keys in registers when M <= 256; ties at the threshold go to the
//        smaller block index, and the selected indices are compacted in ascending order
//        with ordered ballots.
// Token padding: the pooled query of a block averages its real rows only, and every
// padded block (fewer than B real tokens) is forced into every list. It takes the key
// +inf in the selection (scores are finite), so the radix select, the tie rule and the
// compaction treat it as the largest score without a separate pass; the scores
// written out keep the real values.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace bsa {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kSeg = 32;                      // rows per pooling segment
constexpr uint32_t kForcedKey = 0x7F800000u;  // bit pattern of +inf
// shared-memory floats of the scoring pass's copy slots: D/32 chunks x 2 rows of 16 bytes
// per thread
template <int D>
constexpr int kKvFloats = 2 * (D / 32) * kThreads * 4;

// Column sums of every 32-row segment of Q over its real rows: partial[bh][seg][D].
template <int B, int D>
__global__ void __launch_bounds__(kThreads)
k_pool(const __nv_bfloat16* __restrict__ Q, const int32_t* __restrict__ key_valid, int L,
       int n_seg_total, float* __restrict__ partial, int32_t* status) {
  constexpr int CPR = D / 8;          // 16-byte chunks per row
  constexpr int RPI = 32 / CPR;       // rows per warp iteration
  constexpr int NIT = kSeg / RPI;     // iterations per segment (all loads in flight)
  const int lane = threadIdx.x % 32;
  const int cc = lane % CPR, r0 = lane / CPR;
  const int segs_per_head = L / kSeg;
  const int warps = gridDim.x * kWarps;
  for (int sg = blockIdx.x * kWarps + threadIdx.x / 32; sg < n_seg_total; sg += warps) {
    const int bh = sg / segs_per_head, s = sg % segs_per_head;
    const int row0 = s * kSeg;          // first row of the segment within the head
    int nq = kSeg;                      // real rows of the segment
    if (key_valid != nullptr) {
      const int blk = row0 / B;
      const int raw = __ldg(key_valid + blk);
      if ((raw < 1 || raw > B) && lane == 0 && row0 % B == 0) report(status, BSA_ERR_BAD_PADDING);
      const int v = min(max(raw, 1), B);
      nq = min(kSeg, max(0, v - (row0 - blk * B)));
    }
    const uint4* src = reinterpret_cast<const uint4*>(Q + ((size_t)bh * L + row0) * D) + cc;
    uint4 u[NIT];
#pragma unroll
    for (int it = 0; it < NIT; ++it) u[it] = __ldg(src + (size_t)(it * RPI + r0) * CPR);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int it = 0; it < NIT; ++it) {
      if (it * RPI + r0 < nq) {
        float f[8];
        bf16x8_to_f32(u[it], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += f[e];
      }
    }
#pragma unroll
    for (int o = CPR; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    if (lane < CPR) {
      float4* dst = reinterpret_cast<float4*>(partial + (size_t)sg * D + cc * 8);
      dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
}

// Scores of the CTA's kWarps pooled queries (s_q, kWarps x D) against the head's M
// centroids kb (M x D): s_sc[w][j] = scale * s_q[w] . kb[j]. Eight lanes share one
// centroid row: lane g of the group takes the 16-byte chunks g, g + 8, g + 16, ... of the
// row, so each load instruction of a warp reads four rows in whole 128-byte segments; the
// eight partial dots are added across the group by a butterfly, after which lane g holds
// query w = g's score.
// Wait until at most n of this thread's copy groups are pending (n a compile-time value).
__device__ __forceinline__ void cp_async_wait(int n) {
  switch (n) {
    case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
  }
}

template <int D>
__device__ __forceinline__ void score_block(const float* __restrict__ kb, bool vec, int M,
                                            float scale, const float* s_q, float* s_sc,
                                            float4* s_kv, int warp, int lane) {
  constexpr int kG = 8;                 // lanes per centroid
  constexpr int kSub = 32 / kG;         // lane groups of a warp
  constexpr int kRowsWarp = 2 * kSub;   // centroids per warp pass: two per lane
  constexpr int kRowsCta = kWarps * kRowsWarp;
  constexpr int kIt = D / (4 * kG);     // 16-byte chunks per lane per row
  static_assert(kWarps == kG, "lane g of a group writes query block g");
  static_assert(kIt <= 4, "copy-group waits");
  const int g = lane % kG, rsub = lane / kG;
  const int n_pass = (M - warp * kRowsWarp + kRowsCta - 1) / kRowsCta;
  // Lane (g, rsub) takes rows rsub and rsub + kSub of each warp pass, so that every chunk
  // of a pooled query read from shared memory serves two rows. With 16-byte aligned rows
  // the chunks are copied (cp.async) into the thread's own slots of shared memory (s_kv:
  // kIt chunks x 2 rows per thread, thread-major), one copy group per chunk: the next
  // pass's chunk goes into the slots of this pass's chunk as soon as its arithmetic has
  // consumed them. A thread reads back only what it copied itself: no barrier, only its
  // own waits for its copy groups.
  auto row_of = [&](int ps, int h) { return warp * kRowsWarp + ps * kRowsCta + rsub + h * kSub; };
  auto copy_chunk = [&](int ps, int it) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = row_of(ps, h);
      const float* kr = kb + (size_t)(j < M ? j : 0) * D;
      const uint32_t dst = static_cast<uint32_t>(
          __cvta_generic_to_shared(s_kv + (it * 2 + h) * kThreads + threadIdx.x));
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst),
                   "l"(kr + (it * kG + g) * 4)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  if (vec && n_pass > 0) {
#pragma unroll
    for (int it = 0; it < kIt; ++it) copy_chunk(0, it);
  }
  for (int ps = 0; ps < n_pass; ++ps) {
    const bool more = ps + 1 < n_pass;
    float acc0[kWarps], acc1[kWarps];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) acc0[w] = acc1[w] = 0.f;
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
      const int c = (it * kG + g) * 4;
      float4 k0, k1;
      if (vec) {
        // newer groups than this chunk's: this pass's later chunks, and (unless this is
        // the last pass) the next pass's earlier chunks
        cp_async_wait(more ? kIt - 1 : kIt - 1 - it);
        k0 = s_kv[(it * 2) * kThreads + threadIdx.x];
        k1 = s_kv[(it * 2 + 1) * kThreads + threadIdx.x];
      } else {
        const int j0 = row_of(ps, 0), j1 = row_of(ps, 1);
        const float* r0 = kb + (size_t)(j0 < M ? j0 : 0) * D + c;
        const float* r1 = kb + (size_t)(j1 < M ? j1 : 0) * D + c;
        k0 = make_float4(__ldg(r0), __ldg(r0 + 1), __ldg(r0 + 2), __ldg(r0 + 3));
        k1 = make_float4(__ldg(r1), __ldg(r1 + 1), __ldg(r1 + 2), __ldg(r1 + 3));
      }
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float4 qv = *reinterpret_cast<const float4*>(s_q + w * D + c);
        acc0[w] = fmaf(qv.w, k0.w, fmaf(qv.z, k0.z, fmaf(qv.y, k0.y, fmaf(qv.x, k0.x, acc0[w]))));
        acc1[w] = fmaf(qv.w, k1.w, fmaf(qv.z, k1.z, fmaf(qv.y, k1.y, fmaf(qv.x, k1.x, acc1[w]))));
      }
      // the slots of this chunk are consumed: refill them. The empty asm takes the loaded
      // values as inputs, so the loads have completed before the copy is issued
      if (vec && more) {
        asm volatile("" ::"f"(k0.x), "f"(k0.y), "f"(k0.z), "f"(k0.w), "f"(k1.x), "f"(k1.y),
                     "f"(k1.z), "f"(k1.w)
                     : "memory");
        copy_chunk(ps + 1, it);
      }
    }
#pragma unroll
    for (int o = 1; o < kG; o <<= 1)
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        acc0[w] += __shfl_xor_sync(0xffffffffu, acc0[w], o);
        acc1[w] += __shfl_xor_sync(0xffffffffu, acc1[w], o);
      }
    float mine0 = acc0[0], mine1 = acc1[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
      if (g == w) {
        mine0 = acc0[w];
        mine1 = acc1[w];
      }
    }
    const int j0 = row_of(ps, 0), j1 = row_of(ps, 1);
    if (j0 < M) s_sc[g * M + j0] = scale * mine0;
    if (j1 < M) s_sc[g * M + j1] = scale * mine1;
  }
}

// The threshold of the k largest of NK * 32 keys held in registers (key j = lane + 32 q;
// keys of absent j are 0) by a bitwise radix select: from the top bit down, T keeps a bit
// when at least k keys are >= T with it set. Bit 31 is the sign, 0 for every key. Every
// candidate has a bit set, so keys of 0 are never counted. The select stops as soon as
// exactly k keys are >= T: they are then the k largest, whatever the lower bits (T is the
// k-th largest key itself when it runs to the last bit).
template <int NK>
__device__ __forceinline__ uint32_t select_kth(const uint32_t (&key)[NK], int k_top) {
  uint32_t T = 0;
  for (int bit = 30; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    int cnt = 0;
#pragma unroll
    for (int q = 0; q < NK; ++q) cnt += key[q] >= cand ? 1 : 0;
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= k_top) {
      T = cand;
      if (cnt == k_top) break;
    }
  }
  return T;
}

// NK > 0: M <= 32 NK, and each lane keeps its scores (j = lane + 32 q) in registers from
// the softmax to the compaction. NK == 0: any M, scores in shared memory.
template <int B, int D, int NK>
__global__ void __launch_bounds__(kThreads, 5)
k_route(const float* __restrict__ partial, const float* __restrict__ kbar,
        const float* __restrict__ Mnorm, const int32_t* __restrict__ key_valid, int L,
        int k_top, float lambda, float scale, int32_t* __restrict__ row_ptr,
        int32_t* __restrict__ col_idx, float* __restrict__ scores, int32_t* status) {
  const int M = L / B;
  const int bh = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int i = blockIdx.x * kWarps + warp;  // this warp's query block
  const bool active = i < M;

  extern __shared__ __align__(16) float smem[];
  float4* s_kv = reinterpret_cast<float4*>(smem);  // centroid chunks in flight, per thread
  float* s_q = smem + kKvFloats<D>;             // kWarps x D (16-byte aligned rows)
  float* s_cov = s_q + kWarps * D;              // M
  float* s_sc = s_cov + M;                      // kWarps x M
  float* s_red = s_sc + kWarps * M;             // kWarps

  // 1. the loads of the covariance terms and of the block's segment sums, all issued
  //    before any is used
  const float* mn = Mnorm + (size_t)bh * M;
  float mpart = 0.f;
  for (int j = threadIdx.x; j < M; j += kThreads) mpart += __ldg(mn + j);
  constexpr int kSegs = B / kSeg;
  const float* ps = partial + ((size_t)bh * (L / kSeg) + (size_t)(active ? i : 0) * kSegs) * D;
  float qs[D / 32];
#pragma unroll
  for (int t = 0; t < D / 32; ++t) {
    float sum = 0.f;
#pragma unroll
    for (int s = 0; s < kSegs; ++s) sum += __ldg(ps + s * D + t * 32 + lane);
    qs[t] = sum;
  }
  int nq = B;  // real rows of block i
  if (key_valid != nullptr && active) nq = min(max(__ldg(key_valid + i), 1), B);

  // normalised covariance term, shared by every query block of the head
  mpart = warp_sum(mpart);
  if (lane == 0) s_red[warp] = mpart;
  // pooled query of block i: the mean of its real rows (zero for an idle warp, which
  // keeps the dots below finite)
  const float inv = active ? 1.0f / (float)nq : 0.f;
  float* qbar = s_q + warp * D;
#pragma unroll
  for (int t = 0; t < D / 32; ++t) qbar[t * 32 + lane] = active ? qs[t] * inv : 0.f;
  __syncthreads();
  float msum = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) msum += s_red[w];
  const float cov = msum > 0.f ? lambda / msum : 0.f;
  for (int j = threadIdx.x; j < M; j += kThreads) s_cov[j] = cov * __ldg(mn + j);

  // 2. block scores a_j = scale * qbar_w . kbar_j for the CTA's query blocks. The rows
  //    are copied to shared memory 16 bytes at a time when the caller's kbar is 16-byte
  //    aligned (each head's slice then is too, since M * D * 4 is a multiple of 16), and
  //    read with scalar loads otherwise
  const bool vec = (reinterpret_cast<uintptr_t>(kbar) & 15u) == 0;
  score_block<D>(kbar + (size_t)bh * M * D, vec, M, scale, s_q, s_sc, s_kv, warp, lane);
  __syncthreads();
  if (!active) return;

  // 3. softmax over the M blocks plus the covariance term; padded blocks take the key +inf
  const float* sc = s_sc + warp * M;
  float* srow = scores ? scores + ((size_t)bh * M + i) * M : nullptr;
  const int64_t base = (int64_t)bh * M * k_top + (int64_t)i * k_top;
  const unsigned lt = (1u << lane) - 1u;
  if constexpr (NK > 0) {
    float x[NK];
    float mx = -INFINITY;
#pragma unroll
    for (int q = 0; q < NK; ++q) {
      const int j = lane + 32 * q;
      x[q] = j < M ? sc[j] : -INFINITY;
      mx = fmaxf(mx, x[q]);
    }
    mx = warp_max(mx);
    float se = 0.f;
#pragma unroll
    for (int q = 0; q < NK; ++q) {
      x[q] = lane + 32 * q < M ? expf(x[q] - mx) : 0.f;
      se += x[q];
    }
    se = warp_sum(se);
    const float inv_se = 1.0f / se;
    uint32_t key[NK];
    int n_forced = 0;
#pragma unroll
    for (int q = 0; q < NK; ++q) {
      const int j = lane + 32 * q;
      key[q] = 0u;
      if (j < M) {
        const float v = x[q] * inv_se + s_cov[j];
        const bool forced = key_valid != nullptr && __ldg(key_valid + j) < B;
        n_forced += forced ? 1 : 0;
        key[q] = forced ? kForcedKey : __float_as_uint(v);
        if (srow) srow[j] = v;
      }
    }
    n_forced = __reduce_add_sync(0xffffffffu, n_forced);
    if (n_forced > k_top) {
      // the list cannot hold every padded block: report, and emit a valid list anyway
      if (lane == 0) report(status, BSA_ERR_BAD_PADDING);
#pragma unroll
      for (int q = 0; q < NK; ++q)
        if (key[q] == kForcedKey) key[q] = 0u;
    }

    // 4. the threshold of the k largest keys, then 5. the ascending compaction: selected =
    //    key > T, or key == T among the first ties_needed such keys in index order
    const uint32_t T = select_kth<NK>(key, k_top);
    int greater = 0;
#pragma unroll
    for (int q = 0; q < NK; ++q) greater += key[q] > T ? 1 : 0;
    greater = __reduce_add_sync(0xffffffffu, greater);
    const int ties_needed = k_top - greater;  // >= 0
    int ties_seen = 0, out = 0;
#pragma unroll
    for (int q = 0; q < NK; ++q) {
      const int j = lane + 32 * q;
      const bool tie = j < M && key[q] == T;
      const unsigned tb = __ballot_sync(0xffffffffu, tie);
      const bool sel = j < M && (key[q] > T || (tie && ties_seen + __popc(tb & lt) < ties_needed));
      const unsigned sb = __ballot_sync(0xffffffffu, sel);
      if (sel) col_idx[base + out + __popc(sb & lt)] = j;
      ties_seen += __popc(tb);
      out += __popc(sb);
    }
  } else {
    float* scw = s_sc + warp * M;
    float mx = -INFINITY;
    for (int j = lane; j < M; j += 32) mx = fmaxf(mx, scw[j]);
    mx = warp_max(mx);
    float se = 0.f;
    for (int j = lane; j < M; j += 32) se += expf(scw[j] - mx);
    se = warp_sum(se);
    const float inv_se = 1.0f / se;
    int n_forced = 0;
    for (int j = lane; j < M; j += 32) {
      const float v = expf(scw[j] - mx) * inv_se + s_cov[j];
      const bool forced = key_valid != nullptr && __ldg(key_valid + j) < B;
      n_forced += forced ? 1 : 0;
      scw[j] = forced ? __uint_as_float(kForcedKey) : v;
      if (srow) srow[j] = v;
    }
    n_forced = __reduce_add_sync(0xffffffffu, n_forced);
    if (n_forced > k_top) {
      if (lane == 0) report(status, BSA_ERR_BAD_PADDING);
      for (int j = lane; j < M; j += 32)
        if (__float_as_uint(scw[j]) == kForcedKey) scw[j] = 0.f;
    }
    __syncwarp();
    // 4. the threshold of the k largest keys by a bitwise radix select over shared memory:
    //    from the top bit down, keep a bit of T when at least k keys are >= T with it set,
    //    and stop once exactly k keys are >= T
    uint32_t T = 0;
    for (int bit = 30; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      int cnt = 0;
      for (int j = lane; j < M; j += 32) cnt += __float_as_uint(scw[j]) >= cand ? 1 : 0;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (cnt >= k_top) {
        T = cand;
        if (cnt == k_top) break;
      }
    }
    int greater = 0;
    for (int j = lane; j < M; j += 32) greater += __float_as_uint(scw[j]) > T ? 1 : 0;
    greater = __reduce_add_sync(0xffffffffu, greater);
    const int ties_needed = k_top - greater;  // >= 0
    // 5. ascending compaction
    int ties_seen = 0, out = 0;
    for (int j0 = 0; j0 < M; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t key = j < M ? __float_as_uint(scw[j]) : 0u;
      const bool tie = j < M && key == T;
      const unsigned tb = __ballot_sync(0xffffffffu, tie);
      const bool sel = j < M && (key > T || (tie && ties_seen + __popc(tb & lt) < ties_needed));
      const unsigned sb = __ballot_sync(0xffffffffu, sel);
      if (sel) col_idx[base + out + __popc(sb & lt)] = j;
      ties_seen += __popc(tb);
      out += __popc(sb);
    }
  }
  if (lane == 0) {
    int32_t* rp = row_ptr + (size_t)bh * (M + 1);
    rp[i] = (int32_t)base;
    if (i == M - 1) rp[M] = (int32_t)((int64_t)bh * M * k_top + (int64_t)M * k_top);
  }
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int B, int D>
cudaError_t run(const Shape& s, const void* Q, const float* kbar, const float* Mnorm,
                int k_top, float lambda, float scale, int32_t* row_ptr, int32_t* col_idx,
                float* scores, void* ws, int32_t* status, cudaStream_t st) {
  const int M = s.M();
  float* partial = static_cast<float*>(ws);
  // pooling: as many CTAs as are resident at once, each warp looping over 32-row
  // segments (one wave, no tail of late CTAs)
  const int n_seg = s.BH() * (s.L / kSeg);
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_pool<B, D>, kThreads, 0);
  if (e != cudaSuccess) return e;
  const int pool_grid = std::min(ceil_div(n_seg, kWarps), std::max(per_sm, 1) * sm_count());
  k_pool<B, D><<<pool_grid, kThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(Q), s.key_valid,
                                               s.L, n_seg, partial, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t sm =
      ((size_t)kKvFloats<D> + kWarps * D + M + (size_t)kWarps * M + kWarps) * sizeof(float);
  const dim3 grid(ceil_div(M, kWarps), s.BH());
  auto go = [&](auto kern) -> cudaError_t {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (err != cudaSuccess) return err;
    // five CTAs of the scoring kernel per SM (one wave at 40 heads of 128 blocks) need
    // most of the SM's shared memory
    err = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    if (err != cudaSuccess) return err;
    kern<<<grid, kThreads, sm, st>>>(partial, kbar, Mnorm, s.key_valid, s.L, k_top, lambda, scale,
                                     row_ptr, col_idx, scores, status);
    return cudaSuccess;
  };
  if (M <= 128) e = go(k_route<B, D, 4>);
  else if (M <= 256) e = go(k_route<B, D, 8>);
  else e = go(k_route<B, D, 0>);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

size_t route_workspace(const Shape& s) {
  // one column sum of d floats per 32-row segment of Q
  return (size_t)s.BH() * (s.L / kSeg) * s.d * sizeof(float);
}

cudaError_t launch_route(const Shape& s, const void* Q, const float* kbar, const float* Mnorm,
                         int k_top, float lambda, float scale, int32_t* row_ptr,
                         int32_t* col_idx, float* scores, void* ws, int32_t* status,
                         cudaStream_t st) {
  if (s.block == 64 && s.d == 64)
    return run<64, 64>(s, Q, kbar, Mnorm, k_top, lambda, scale, row_ptr, col_idx, scores, ws,
                       status, st);
  if (s.block == 64 && s.d == 128)
    return run<64, 128>(s, Q, kbar, Mnorm, k_top, lambda, scale, row_ptr, col_idx, scores, ws,
                        status, st);
  if (s.block == 128 && s.d == 64)
    return run<128, 64>(s, Q, kbar, Mnorm, k_top, lambda, scale, row_ptr, col_idx, scores, ws,
                        status, st);
  return run<128, 128>(s, Q, kbar, Mnorm, k_top, lambda, scale, row_ptr, col_idx, scores, ws,
                       status, st);
}

}  // namespace bsa
