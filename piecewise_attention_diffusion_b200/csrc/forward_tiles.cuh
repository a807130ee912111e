// Pieces shared by the attention kernels: the merged key-block lists of a query tile,
// the per-row softmax helpers on an S row held in registers, and the host-side tensor
// maps (TMA descriptors) of the bf16 operands.
#pragma once
#include <limits.h>

#include "common.cuh"
#include "sm100.cuh"

namespace bsa {
namespace fwdtiles {

using namespace sm100;

#ifndef BSA_POLY_OF8
#define BSA_POLY_OF8 2
#endif
// pairs of exponentials, of every 8 pairs of an exact tile, computed on the FMA pipe
constexpr int kPolyOf8 = BSA_POLY_OF8;

// The key-block lists of the (one or two) query blocks of a tile, merged ascending.
struct Lists {
  const int32_t* col;
  int p0, e0, p1, e1;
  __device__ __forceinline__ int next() {
    const int a = p0 < e0 ? __ldg(col + p0) : INT_MAX;
    const int b = p1 < e1 ? __ldg(col + p1) : INT_MAX;
    const int j = min(a, b);
    if (j == INT_MAX) return -1;
    if (a == j) ++p0;
    if (b == j) ++p1;
    return j;
  }
};

// Lists of query tile qt of head bh: query blocks qt*QBPT (and qt*QBPT + 1 when a tile
// holds two blocks). Per-head lists start at row_ptr + bh*(M+1); a shared list serves
// every head.
template <int QBPT>
__device__ __forceinline__ Lists item_lists(const int32_t* row_ptr, const int32_t* col_idx,
                                            int csr_per_head, int M, int bh, int qt) {
  const int32_t* rp = csr_per_head ? row_ptr + (size_t)bh * (M + 1) : row_ptr;
  const int i0 = qt * QBPT;
  Lists r;
  r.col = col_idx;
  r.p0 = __ldg(rp + i0);
  r.e0 = __ldg(rp + i0 + 1);
  r.p1 = r.e1 = 0;
  if (QBPT == 2 && i0 + 1 < M) {
    r.p1 = r.e0;
    r.e1 = __ldg(rp + i0 + 2);
  }
  return r;
}

// Number of distinct key blocks in a tile's merged lists.
template <int QBPT>
__device__ __forceinline__ int count_exact(Lists l) {
  if (QBPT == 1) return l.e0 - l.p0;
  int n = 0;
  while (l.next() >= 0) ++n;
  return n;
}

// Row max of the first N of the R columns held in registers: three-input max in four
// chains.
template <int N, int R>
__device__ __forceinline__ float row_max(const uint32_t (&r)[R]) {
  static_assert(N <= R && N % 8 == 0, "row_max");
  float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
  for (int e = 0; e < N; e += 8) {
    m0 = max3(m0, __uint_as_float(r[e]), __uint_as_float(r[e + 1]));
    m1 = max3(m1, __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
    m2 = max3(m2, __uint_as_float(r[e + 4]), __uint_as_float(r[e + 5]));
    m3 = max3(m3, __uint_as_float(r[e + 6]), __uint_as_float(r[e + 7]));
  }
  return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}

// Sum of the first N columns held in registers (packed adds in four chains).
template <int N, int R>
__device__ __forceinline__ float row_sum(const uint32_t (&r)[R]) {
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
#pragma unroll
  for (int q = 0; q < N / 2; ++q)
    acc[q & 3] = add2(acc[q & 3], make_float2(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1])));
  const float2 a = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
  return a.x + a.y;
}

// Linear weights c1 * s + c0 for the first N columns in r, written to TMEM as bf16 pairs
// (column c holds elements 2c and 2c + 1) at p_addr.
template <int N, int R>
__device__ __forceinline__ void row_lin(const uint32_t (&r)[R], float c1, float c0,
                                        uint32_t p_addr) {
  const float2 a = make_float2(c1, c1), b = make_float2(c0, c0);
#pragma unroll
  for (int h = 0; h < N / 64; ++h) {
    uint32_t pk[32];
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      const int e = h * 64 + 2 * q;
      const float2 w = fma2(make_float2(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), a, b);
      pk[q] = pack_bf16x2(w.x, w.y);
    }
    tmem_st32(p_addr + h * 32, pk);
  }
}

// P for one row: 2^(s * scale_log2 - m_ref) for the first N columns in r, written to TMEM
// as bf16 pairs (column c holds elements 2c and 2c + 1) at p_addr; returns the fp32 row
// sum. With kMixed, kPolyOf8 of every 8 pairs are computed on the FMA pipe (ex2_poly2)
// and the rest on the special-function unit, so that the two pipes share the work; a row
// that may hold -inf (masked entries) uses the special-function unit only.
template <int N, bool kMixed, int R>
__device__ __forceinline__ float row_exp(const uint32_t (&r)[R], float scale_log2,
                                         float m_ref, uint32_t p_addr) {
  const float2 sc = make_float2(scale_log2, scale_log2);
  const float2 nm = make_float2(-m_ref, -m_ref);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
#pragma unroll
  for (int h = 0; h < N / 64; ++h) {
    uint32_t pk[32];
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      const int e = h * 64 + 2 * q;
      const float2 xx =
          fma2(make_float2(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), sc, nm);
      float2 ev;
      if (kMixed && (q % 8) < kPolyOf8) {
        ev = ex2_poly2(xx);
      } else {
        ev = make_float2(ex2(xx.x), ex2(xx.y));
      }
      acc[q & 3] = add2(acc[q & 3], ev);
      pk[q] = pack_bf16x2(ev.x, ev.y);
    }
    tmem_st32(p_addr + h * 32, pk);
  }
  const float2 a = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
  return a.x + a.y;
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// bf16 tensor [z][rows][cols] (cols contiguous, cols a multiple of 64) viewed as 4-D
// (64 columns, rows, cols/64 column groups, z) so that one box of 64 x box_rows x
// cols/64 lands in shared memory as cols/64 consecutive [box_rows x 64] sub-tiles, each
// 128-byte swizzled: the operand layout of the MMA descriptors (sub-tile h at byte
// offset h * box_rows * 128). With all_groups false the box holds one column group, for
// callers that place the groups themselves (a Q tile shorter than 128 rows).
inline bool make_map(CUtensorMap* m, const void* ptr, int cols, int rows, int z, int box_rows,
                     bool all_groups = true) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {64, (cuuint64_t)rows, (cuuint64_t)(cols / 64), (cuuint64_t)z};
  cuuint64_t strides[3] = {(cuuint64_t)cols * 2, 128, (cuuint64_t)cols * rows * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)box_rows, all_groups ? (cuuint32_t)(cols / 64) : 1u, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace fwdtiles
}  // namespace bsa
