// bsa_precompute on the tensor cores (tcgen05 + TMEM + TMA), sm_100a, head dim 64 and 128.
//
// "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers",
// technical summary §2: per KV block j the centroid kbar_j, the value sum vsum_j and
// the first-order matrix H_j = sum_n (k_{j,n} - kbar_j)^T v_{j,n}; H-bar is the mean of
// the H_j over the head and routing uses M_j = ||H_j - H-bar||.
//
// Per block the tensor core computes, from the K_j and V_j tiles exactly as TMA lands
// them (both operands MN-major, 128-byte swizzled; a head dimension of 64 is padded to
// 128 in shared memory by a second 64-column sub-tile of zeros that TMA never writes, so
// the products are the d = 128 ones with zero rows and columns past 64, and only the
// real 64 x 64 corner is written out):
//     C_j    = K_j^T V_j                  (d x d, fp32 in TMEM)
//     ksum_j = K_j^T 1,  vsum_j = V_j^T 1  (against a tile of ones: exact column sums)
// and the epilogue thread that owns row a of C applies the centring in fp32:
//     H_j[a][c] = C_j[a][c] - (ksum_j[a] / B) * vsum_j[c].
// Two passes over K and V, because M_j needs H-bar, i.e. every block of the head:
//   stats pass  writes kbar, vsum and, per head segment of its range, the partial sum
//               of H_j (rows kept in registers; written once per segment);
//   (a reduce kernel then forms H-bar from the partials in a fixed order; the norm pass
//   is launched as its programmatic dependent, so that the norm pass's K/V stream starts
//   while H-bar is formed, and only its epilogue waits for the reduce);
//   norm pass   recomputes H_j and reduces ||H_j - H-bar||_F over the 128 rows.
// Each pass is one persistent kernel; the flattened (head, block) range is dealt in
// contiguous pieces of equal length, one per CTA (so every SM works, and a CTA meets
// few heads and reloads H-bar rarely): warp 0 issues TMA into a 3-stage ring of (K_j,
// V_j) pairs, warp 1 issues the MMAs into two TMEM buffers, warps 2-5 run the epilogue.
// Every mbarrier wait is bounded; a timeout aborts the CTA and reports BSA_ERR_TIMEOUT.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace bsa {
namespace pretc {

using namespace sm100;

constexpr int D = 128;
constexpr int kThreads = 192;
constexpr int kStages = 3;
constexpr int kMaxGrid = 256;  // CTAs per pass at most (bounds the partial-sum workspace)
constexpr uint32_t kTmemCols = 512;
// TMEM buffer b: C at 256 b, ksum at 256 b + 128, vsum at 256 b + 144 (16 columns each)

template <int B>
struct Cfg {
  static constexpr int TILE = B * D * 2;       // one K or V tile
  static constexpr int STAGE = 2 * TILE;       // K and V
  static constexpr int ONES = 16 * B * 2;      // 16 x B tile of ones (K-major)
  static constexpr int SMEM = kStages * STAGE + ONES + 1024;
};

struct Params {
  int L, M, BH;
  int n_units, per_cta;   // units = blocks (b*H + h) * M + j; CTA c takes [c per_cta, ..)
  bool stats;
  float* kbar;
  float* vsum;
  float* partial;         // stats: slot c + bh per (CTA c, head bh) segment, [., D, D]
  const float* Hbar;      // norm
  float* Mnorm;           // norm
  float* Hblk;            // norm, nullable
  const int32_t* key_valid;  // real tokens per block, or null (no padding)
  int32_t* status;
};

// The blocks this CTA processes, in order: the contiguous range [u0, u1) of the pass,
// ascending in the statistics pass and descending in the norm pass, so that the norm pass
// starts on the blocks the statistics pass read last (still in L2).
// A head segment is the run of the range's blocks that belong to one head.
struct BlockIter {
  int u, u0, u1, j, bh, M;
  bool down;
  __device__ __forceinline__ void init(const Params& p) {
    M = p.M;
    u0 = blockIdx.x * p.per_cta;
    u1 = min(p.n_units, u0 + p.per_cta);
    down = !p.stats;
    u = down ? u1 - 1 : u0;
    bh = u / M;
    j = u % M;
  }
  __device__ __forceinline__ bool valid() const { return down ? u >= u0 : u < u1; }
  // advance to the next block; returns true when a head segment just ended (used by
  // the ascending statistics pass)
  __device__ __forceinline__ bool next() {
    if (down) {
      --u;
      if (--j < 0) {
        j = M - 1;
        --bh;
        return true;
      }
      return u < u0;
    }
    ++u;
    ++j;
    if (j == M) {
      j = 0;
      ++bh;
      return true;
    }
    return u >= u1;
  }
};

struct Barriers {
  uint64_t full[kStages], empty[kStages];
  uint64_t mma_done[2], tmem_free[2], xch[2], xred[2];
  uint64_t done;
};

template <int B, int DO, bool kStats>
__global__ void __launch_bounds__(kThreads, 1)
k_precompute(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
             const Params p) {
  using C = Cfg<B>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sOnes = smem + kStages * C::STAGE;
  __shared__ Barriers bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float s_vs[2][D];
  __shared__ float s_red[2][4];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // ones tile (its swizzle is irrelevant: every element is 1.0)
  for (int e = threadIdx.x; e < C::ONES / 4; e += kThreads)
    reinterpret_cast<uint32_t*>(sOnes)[e] = 0x3F803F80u;  // bf16 pair (1.0, 1.0)
  if constexpr (DO < D) {
    // head dimension 64: the second 64-column sub-tile of every K and V tile stays zero
    for (int t = 0; t < 2 * kStages; ++t) {
      uint4* z = reinterpret_cast<uint4*>(smem + t * C::TILE + B * 128);
      for (int e = threadIdx.x; e < B * 128 / 16; e += kThreads) z[e] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bars.full[i], 1);
      mbar_init(&bars.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.mma_done[i], 1);
      mbar_init(&bars.tmem_free[i], 128);
      mbar_init(&bars.xch[i], 128);
      mbar_init(&bars.xred[i], 128);
    }
    mbar_init(&bars.done, 1);
    fence_barrier_init();
  }
  // the ones tile is read by the tensor core (async proxy)
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;

  if (warp == 0) {
    // ============================================================== TMA producer
    if (lane == 0) {
      BlockIter it;
      it.init(p);
      uint32_t n = 0;
      bool ok = true;
      while (it.valid()) {
        const int st = n % kStages;
        if (!(ok = mbar_wait(&bars.empty[st], ((n / kStages) & 1) ^ 1, abort_flag))) break;
        unsigned char* dst = smem + st * C::STAGE;
        mbar_arrive_expect_tx(&bars.full[st], 2u * B * DO * 2u);  // K and V, real columns
        tma_load_4d(dst, &tmK, &bars.full[st], 0, it.j * B, 0, it.bh);
        tma_load_4d(dst + C::TILE, &tmV, &bars.full[st], 0, it.j * B, 0, it.bh);
        ++n;
        it.next();
      }
      if (!ok) {
        const uint64_t t0 = globaltimer_ns();
        const uint32_t first = n > (uint32_t)kStages ? n - kStages : 0;
        for (uint32_t r = first; r < n; ++r)
          while (!mbar_try_wait(&bars.full[r % kStages], (r / kStages) & 1) &&
                 globaltimer_ns() - t0 < 100000000ull) {
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    // Lane 0 issues; with token padding the whole warp first zeroes the tail rows of a
    // padded block's K and V tiles, so that every product and column sum runs over the
    // real tokens only (a row fills 128 bytes of each 64-column sub-tile, whatever the
    // swizzle).
    constexpr uint32_t idesc_c = idesc_bf16_f32(128, D, true, true);
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, 16, true, false);
    const uint32_t ones = smem_u32(sOnes);
    BlockIter it;
    it.init(p);
    uint32_t n = 0;
    bool ok = true;
    while (it.valid()) {
      const int st = n % kStages, b = n & 1;
      ok = mbar_wait(&bars.full[st], (n / kStages) & 1, abort_flag);
      if (ok && n >= 2) ok = mbar_wait(&bars.tmem_free[b], ((n >> 1) - 1) & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      unsigned char* stage = smem + st * C::STAGE;
      if (p.key_valid != nullptr) {
        const int v = min(max(__ldg(p.key_valid + it.j), 1), B);
        if (v < B) {
          constexpr int kChunks = (DO / 64) * 8;  // 16-byte chunks of one row's real columns
          for (int e = lane; e < 2 * (B - v) * kChunks; e += 32) {
            const int tile = e / ((B - v) * kChunks), rest = e % ((B - v) * kChunks);
            const int r = v + rest / kChunks, c = rest % kChunks;
            *reinterpret_cast<uint4*>(stage + tile * C::TILE + (c / 8) * (B * 128) + r * 128 +
                                      (c % 8) * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          // the tensor core (async proxy) reads what these generic stores wrote
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
        }
      }
      if (lane == 0) {
        tc_fence_after();
        const uint32_t k_addr = smem_u32(stage);
        const uint32_t v_addr = k_addr + C::TILE;
        const uint32_t dc = tmem + 256u * b;
#pragma unroll
        for (int k = 0; k < B / 16; ++k) {
          const uint64_t a_k = smem_desc_sw128(k_addr + k * 2048, B * 128, 1024);
          const uint64_t a_v = smem_desc_sw128(v_addr + k * 2048, B * 128, 1024);
          const uint64_t b_o = smem_desc_sw128(ones + (k / 4) * (16 * 128) + (k % 4) * 32, 16, 1024);
          mma_ss(dc, a_k, a_v, idesc_c, k > 0 ? 1u : 0u);          // K^T V
          mma_ss(dc + 128, a_k, b_o, idesc_s, k > 0 ? 1u : 0u);    // K^T 1
          mma_ss(dc + 144, a_v, b_o, idesc_s, k > 0 ? 1u : 0u);    // V^T 1
        }
        mma_commit(&bars.empty[st]);
        mma_commit(&bars.mma_done[b]);
      }
      __syncwarp();
      ++n;
      it.next();
    }
    if (lane == 0) {
      mma_commit(&bars.done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&bars.done, 0) && globaltimer_ns() - t0 < 100000000ull) {
      }
    }
    __syncwarp();
  } else {
    // ================================================================== epilogue
    const int quad = warp % 4;
    const int a = quad * 32 + lane;              // row of C = TMEM lane
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    // stats: partial sum of H_j row a over the head segment; norm: H-bar row a of the head
    // (rows a >= DO of a padded head dimension are zero throughout and write nothing)
    float acc[DO];
#pragma unroll
    for (int c = 0; c < DO; ++c) acc[c] = 0.f;
    int hb_head = -1;
    // norm pass: H-bar comes from the reduce kernel, which this grid may overlap
    // (programmatic dependent launch): wait for it to complete before the first read
    if (!kStats) asm volatile("griddepcontrol.wait;" ::: "memory");
    BlockIter it;
    it.init(p);
    uint32_t n = 0;
    bool ok = true;
    while (it.valid()) {
      const int b = n & 1;
      const uint32_t ph = (n >> 1) & 1;
      const int bh = it.bh, j = it.j;
      if (!kStats && bh != hb_head) {
        if (a < DO) {
          const float4* src =
              reinterpret_cast<const float4*>(p.Hbar + ((size_t)bh * DO + a) * DO);
#pragma unroll
          for (int c = 0; c < DO / 4; ++c) {
            const float4 v = __ldg(src + c);
            acc[4 * c] = v.x;
            acc[4 * c + 1] = v.y;
            acc[4 * c + 2] = v.z;
            acc[4 * c + 3] = v.w;
          }
        }
        hb_head = bh;
      }
      ok = mbar_wait(&bars.mma_done[b], ph, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t base = tmem + lane_addr + 256u * b;
      float kb, vs;
      {
        uint32_t r0[16], r1[16];
        tmem_ld16(base + 128, r0);
        tmem_ld16(base + 144, r1);
        tmem_wait_ld();
        int nv = B;  // real tokens of the block
        if (p.key_valid != nullptr) {
          const int raw = __ldg(p.key_valid + j);
          if ((raw < 1 || raw > B) && a == 0) report(p.status, BSA_ERR_BAD_PADDING);
          nv = min(max(raw, 1), B);
        }
        kb = __uint_as_float(r0[0]) / (float)nv;
        vs = __uint_as_float(r1[0]);
      }
      if (kStats && a < DO) {
        const size_t o = ((size_t)bh * p.M + j) * DO + a;
        p.kbar[o] = kb;
        p.vsum[o] = vs;
      }
      // every row needs vsum_j[c] for all c: exchange through shared memory
      s_vs[b][a] = vs;
      mbar_arrive(&bars.xch[b]);
      ok = mbar_wait(&bars.xch[b], ph, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      float sq = 0.f;
      float* hrow = (!kStats && p.Hblk && a < DO)
                        ? p.Hblk + (((size_t)bh * p.M + j) * DO + a) * DO
                        : nullptr;
#pragma unroll
      for (int c0 = 0; c0 < DO; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(base + c0, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float h = fmaf(-kb, s_vs[b][c0 + e], __uint_as_float(r[e]));
          if (kStats) {
            acc[c0 + e] += h;
          } else {
            const float dlt = h - acc[c0 + e];
            sq = fmaf(dlt, dlt, sq);
            r[e] = __float_as_uint(h);
          }
        }
        if (hrow) {
          float4* dst = reinterpret_cast<float4*>(hrow + c0);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                 __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
        }
      }
      // the TMEM buffer is free for the block after next
      tc_fence_before();
      mbar_arrive(&bars.tmem_free[b]);
      if (!kStats) {
        sq = warp_sum(sq);
        if (lane == 0) s_red[b][quad] = sq;
        mbar_arrive(&bars.xred[b]);
        ok = mbar_wait(&bars.xred[b], ph, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (a == 0)
          p.Mnorm[(size_t)bh * p.M + j] =
              sqrtf((s_red[b][0] + s_red[b][1]) + (s_red[b][2] + s_red[b][3]));
      }
      ++n;
      const bool unit_end = it.next();
      if (kStats && unit_end) {
        // head segment finished: write its partial sum (row a) into slot blockIdx.x + bh
        // (distinct per (CTA, head): the next CTA's first head is at least this one's
        // last) and start a new one
        float4* dst = reinterpret_cast<float4*>(
            p.partial + (((size_t)blockIdx.x + bh) * DO + a) * DO);
#pragma unroll
        for (int c = 0; c < DO / 4; ++c) {
          if (a < DO)
            dst[c] = make_float4(acc[4 * c], acc[4 * c + 1], acc[4 * c + 2], acc[4 * c + 3]);
          acc[4 * c] = acc[4 * c + 1] = acc[4 * c + 2] = acc[4 * c + 3] = 0.f;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && abort_sh) report(p.status, BSA_ERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// H-bar = (1 / M) * sum of the head's segment partial sums, in CTA order (fixed for a
// given grid: deterministic). CTA c covers blocks [c per, (c + 1) per) of the flattened
// (head, block) range, so head bh's segments come from CTAs bh M / per ..
// ((bh + 1) M - 1) / per, and CTA c wrote its segment of head bh into slot c + bh.
template <int DO>
__global__ void k_reduce(const float* __restrict__ partial, int per, int grid, int M,
                         float* __restrict__ Hbar) {
  // the norm pass may start now (programmatic dependent launch): its TMA and MMA warps
  // read only K and V, and its epilogue waits for this grid before it reads H-bar
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const int bh = blockIdx.y;
  if (e >= DO * DO) return;
  const int c0 = (int)((int64_t)bh * M / per);
  const int c1 = min(grid - 1, (int)(((int64_t)bh * M + M - 1) / per));
  float s = 0.f;
  for (int c = c0; c <= c1; ++c) s += partial[((size_t)c + bh) * DO * DO + e];
  Hbar[(size_t)bh * DO * DO + e] = s / (float)M;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// K or V [BH][L][d] as 4-D (64 columns, L rows, d/64 groups, BH): one box = one block tile
// landing as d/64 swizzled [B x 64] sub-tiles.
bool make_map(CUtensorMap* m, const void* ptr, int L, int BH, int B, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {64, (cuuint64_t)L, (cuuint64_t)(d / 64), (cuuint64_t)BH};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, 128, (cuuint64_t)d * L * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)B, (cuuint32_t)(d / 64), 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int B, int DO>
cudaError_t run(const Shape& s, const void* K, const void* V, float* kbar, float* vsum,
                float* Hbar, float* Mnorm, float* Hblk, void* ws, int32_t* status,
                cudaStream_t st) {
  using Cf = Cfg<B>;
  CUtensorMap tmK, tmV;
  if (!make_map(&tmK, K, s.L, s.BH(), B, DO) || !make_map(&tmV, V, s.L, s.BH(), B, DO))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(k_precompute<B, DO, true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_precompute<B, DO, false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM);
  if (e != cudaSuccess) return e;
  const int M = s.M(), sms = std::min(sm_count(), kMaxGrid);
  Params p;
  p.L = s.L;
  p.M = M;
  p.BH = s.BH();
  p.kbar = kbar;
  p.vsum = vsum;
  p.partial = static_cast<float*>(ws);
  p.Hbar = Hbar;
  p.Mnorm = Mnorm;
  p.Hblk = Hblk;
  p.key_valid = s.key_valid;
  p.status = status;
  // both passes deal the flattened (head, block) range in contiguous pieces, one per CTA
  p.n_units = s.BH() * M;
  p.per_cta = ceil_div(p.n_units, sms);
  const int grid = ceil_div(p.n_units, p.per_cta);
  p.stats = true;
  k_precompute<B, DO, true><<<grid, kThreads, Cf::SMEM, st>>>(tmK, tmV, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_reduce<DO><<<dim3(ceil_div(DO * DO, 256), s.BH()), 256, 0, st>>>(p.partial, p.per_cta,
                                                                       grid, M, Hbar);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  p.stats = false;
  // launched as a programmatic dependent of the reduce kernel, so that its K/V stream
  // starts while H-bar is being formed
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cf::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_precompute<B, DO, false>, tmK, tmV, p);
}

}  // namespace pretc

size_t precompute_workspace(const Shape& s) {
  // one partial sum per (CTA, head) segment: at most grid + BH - 1 slots, grid <= kMaxGrid
  // and <= the number of blocks
  const size_t grid = std::min<size_t>(pretc::kMaxGrid, (size_t)s.BH() * s.M());
  return (grid + s.BH()) * (size_t)s.d * s.d * sizeof(float);
}

cudaError_t launch_precompute(const Shape& s, const void* K, const void* V, float* kbar,
                              float* vsum, float* Hbar, float* Mnorm, float* Hblk, void* ws,
                              int32_t* status, cudaStream_t st) {
  if (s.d == 64) {
    if (s.block == 64)
      return pretc::run<64, 64>(s, K, V, kbar, vsum, Hbar, Mnorm, Hblk, ws, status, st);
    return pretc::run<128, 64>(s, K, V, kbar, vsum, Hbar, Mnorm, Hblk, ws, status, st);
  }
  if (s.block == 64)
    return pretc::run<64, 128>(s, K, V, kbar, vsum, Hbar, Mnorm, Hblk, ws, status, st);
  return pretc::run<128, 128>(s, K, V, kbar, vsum, Hbar, Mnorm, Hblk, ws, status, st);
}

}  // namespace bsa
