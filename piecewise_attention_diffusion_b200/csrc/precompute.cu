// bsa_precompute: per-block statistics of the piecewise (PISA) form.
//
// "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers",
// technical summary §2: before the fused attention pass, compute each KV block's key
// centroid kbar_j and value sum, and the global first-order statistic H-bar = mean over
// blocks of H_j; routing adds M_j = ||H_j - H-bar||.
//
// H_j is computed with the rank-1 identity
//     H_j = sum_n (k_n - kbar_j)^T v_n = K_j^T V_j - kbar_j^T vsum_j,
// so the d x d product K_j^T V_j runs on the tensor cores (bf16 in, fp32 accumulate)
// and the centring is one fp32 rank-1 update. The kernels are HBM-bound (each block's
// K and V are read once per pass); three launches (this file serves d = 64; d = 128
// runs on the tensor-core kernels of precompute_tc.cu):
//   k_pre_stats : kbar, vsum, and partial sums of H_j over groups of G blocks;
//   k_pre_reduce: Hbar = (1/M) * sum of the partials, in a fixed order (deterministic);
//   k_pre_norm  : recompute H_j per block, Mnorm_j = ||H_j - Hbar||_F, optional H_j out.
#include "common.cuh"
#include "internal.h"

namespace bsa {
namespace {

constexpr int kThreads = 256;  // 8 warps

// Shared-memory tile of one block: B rows x D bf16, rows padded by 16 bytes so that
// ldmatrix phases over 8 consecutive rows hit 8 distinct bank quads.
template <int D>
struct TilePitch {
  static constexpr int elems = D + 8;
};

template <int B, int D>
__device__ __forceinline__ void load_tile_async(__nv_bfloat16* dst, const __nv_bfloat16* src) {
  constexpr int chunks_per_row = D / 8;  // 16-byte chunks
  constexpr int total = B * chunks_per_row;
  const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  for (int c = threadIdx.x; c < total; c += kThreads) {
    const int r = c / chunks_per_row, cc = c % chunks_per_row;
    const uint32_t saddr = base + (r * TilePitch<D>::elems + cc * 8) * 2;
    const void* g = src + (size_t)r * D + cc * 8;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(saddr), "l"(g));
  }
  asm volatile("cp.async.commit_group;\n" ::);
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;\n" ::);
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t* r, uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr));
}

__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Warp tiling of the D x D product K^T V over 8 warps (4 along rows a, 2 along cols c).
template <int D>
struct Tiling {
  static constexpr int WM = D / 4, WN = D / 2;
  static constexpr int MT = WM / 16, NT = WN / 8;
};

// acc += Ks^T Vs over the B tokens of one tile (both tiles resident in shared memory).
template <int B, int D>
__device__ __forceinline__ void ktv_accumulate(float (&acc)[Tiling<D>::MT][Tiling<D>::NT][4],
                                               const __nv_bfloat16* Ks,
                                               const __nv_bfloat16* Vs) {
  using T = Tiling<D>;
  constexpr int P = TilePitch<D>::elems;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int a_base = (warp / 2) * T::WM, c_base = (warp % 2) * T::WN;
  const uint32_t ks = static_cast<uint32_t>(__cvta_generic_to_shared(Ks));
  const uint32_t vs = static_cast<uint32_t>(__cvta_generic_to_shared(Vs));
  const int mat = lane / 8, r = lane % 8;
#pragma unroll
  for (int n0 = 0; n0 < B; n0 += 16) {
    uint32_t af[T::MT][4];
#pragma unroll
    for (int mt = 0; mt < T::MT; ++mt) {
      // A = K^T: matrices (tokens 0-7 | 8-15) x (a 0-7 | 8-15), transposed on load.
      const int n_off = (mat >> 1) * 8, a_off = (mat & 1) * 8;
      const int row = n0 + n_off + r, col = a_base + mt * 16 + a_off;
      ldmatrix_x4_trans(af[mt], ks + (row * P + col) * 2);
    }
#pragma unroll
    for (int np = 0; np < T::NT / 2; ++np) {
      // B = V: matrices (tokens 0-7 | 8-15) x (c 0-7 | 8-15) of two n8 tiles.
      const int n_off = (mat & 1) * 8, c_off = (mat >> 1) * 8;
      const int row = n0 + n_off + r, col = c_base + np * 16 + c_off;
      uint32_t bf[4];
      ldmatrix_x4_trans(bf, vs + (row * P + col) * 2);
#pragma unroll
      for (int mt = 0; mt < T::MT; ++mt) {
        mma_bf16_16816(acc[mt][2 * np], af[mt], bf);
        mma_bf16_16816(acc[mt][2 * np + 1], af[mt], bf + 2);
      }
    }
  }
}

// Visit the (a, c) coordinates this thread owns in the accumulator fragments.
template <int D, class F>
__device__ __forceinline__ void for_each_acc(float (&acc)[Tiling<D>::MT][Tiling<D>::NT][4], F f) {
  using T = Tiling<D>;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int a_base = (warp / 2) * T::WM, c_base = (warp % 2) * T::WN;
  const int g = lane / 4, t = lane % 4;
#pragma unroll
  for (int mt = 0; mt < T::MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < T::NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int a = a_base + mt * 16 + g + (e >> 1) * 8;
        const int c = c_base + nt * 8 + 2 * t + (e & 1);
        f(acc[mt][nt][e], a, c);
      }
}

// Token padding: the block's rows past its nv real tokens are zeroed in both resident
// tiles, so that the column sums and K^T V below run over the real tokens only.
template <int B, int D>
__device__ __forceinline__ void zero_padding(__nv_bfloat16* Ks, __nv_bfloat16* Vs, int nv) {
  constexpr int P = TilePitch<D>::elems;
  for (int e = threadIdx.x; e < (B - nv) * D; e += kThreads) {
    const int r = nv + e / D, c = e % D;
    Ks[r * P + c] = __float2bfloat16(0.f);
    Vs[r * P + c] = __float2bfloat16(0.f);
  }
}

// Real tokens of block j (B without padding); an out-of-range count is reported and
// clamped.
template <int B>
__device__ __forceinline__ int real_tokens(const int32_t* key_valid, int j, int32_t* status) {
  if (key_valid == nullptr) return B;
  const int raw = __ldg(key_valid + j);
  if ((raw < 1 || raw > B) && threadIdx.x == 0) report(status, BSA_ERR_BAD_PADDING);
  return min(max(raw, 1), B);
}

// Column means of K and column sums of V of the resident tile (threads 0..2D-1), over
// the block's nv real tokens (the padded rows are zero).
template <int B, int D>
__device__ __forceinline__ void column_stats(const __nv_bfloat16* Ks, const __nv_bfloat16* Vs,
                                             float* s_kbar, float* s_vsum, int nv) {
  constexpr int P = TilePitch<D>::elems;
  const int t = threadIdx.x;
  if (t < 2 * D) {
    const bool is_k = t < D;
    const int c = is_k ? t : t - D;
    const __nv_bfloat16* src = is_k ? Ks : Vs;
    float s = 0.f;
#pragma unroll 8
    for (int n = 0; n < B; ++n) s += __bfloat162float(src[n * P + c]);
    if (is_k)
      s_kbar[c] = s / (float)nv;
    else
      s_vsum[c] = s;
  }
}

template <int B, int D>
__global__ void __launch_bounds__(kThreads)
k_pre_stats(const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V, int L,
            int G, const int32_t* __restrict__ key_valid, float* __restrict__ kbar,
            float* __restrict__ vsum, float* __restrict__ partial, int32_t* status) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int P = TilePitch<D>::elems;
  __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* Vs = Ks + B * P;
  float* s_kbar = reinterpret_cast<float*>(Vs + B * P);
  float* s_vsum = s_kbar + D;

  const int M = L / B;
  const int bh = blockIdx.y, grp = blockIdx.x, n_grp = gridDim.x;
  const size_t head = (size_t)bh * L * D;
  float acc[Tiling<D>::MT][Tiling<D>::NT][4] = {};

  const int j0 = grp * G, j1 = min(M, j0 + G);
  for (int j = j0; j < j1; ++j) {
    load_tile_async<B, D>(Ks, K + head + (size_t)j * B * D);
    load_tile_async<B, D>(Vs, V + head + (size_t)j * B * D);
    cp_async_wait_all();
    __syncthreads();
    const int nv = real_tokens<B>(key_valid, j, status);
    if (nv < B) {
      zero_padding<B, D>(Ks, Vs, nv);
      __syncthreads();
    }
    column_stats<B, D>(Ks, Vs, s_kbar, s_vsum, nv);
    ktv_accumulate<B, D>(acc, Ks, Vs);
    __syncthreads();
    if (threadIdx.x < D) {
      const size_t o = ((size_t)bh * M + j) * D + threadIdx.x;
      kbar[o] = s_kbar[threadIdx.x];
      vsum[o] = s_vsum[threadIdx.x];
    }
    // centring: subtract kbar_j^T vsum_j from the running sum of K_j^T V_j
    for_each_acc<D>(acc, [&](float& x, int a, int c) { x -= s_kbar[a] * s_vsum[c]; });
    __syncthreads();
  }
  float* out = partial + ((size_t)bh * n_grp + grp) * D * D;
  for_each_acc<D>(acc, [&](float& x, int a, int c) { out[a * D + c] = x; });
}

__global__ void k_pre_reduce(const float* __restrict__ partial, int n_grp, int DD, int M,
                             float* __restrict__ Hbar) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const int bh = blockIdx.y;
  if (e >= DD) return;
  const float* p = partial + (size_t)bh * n_grp * DD + e;
  float s = 0.f;
  for (int g = 0; g < n_grp; ++g) s += p[(size_t)g * DD];
  Hbar[(size_t)bh * DD + e] = s / (float)M;
}

template <int B, int D>
__global__ void __launch_bounds__(kThreads)
k_pre_norm(const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V, int L,
           const int32_t* __restrict__ key_valid, const float* __restrict__ Hbar,
           float* __restrict__ Mnorm, float* __restrict__ Hblk, int32_t* status) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int P = TilePitch<D>::elems;
  __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* Vs = Ks + B * P;
  float* s_kbar = reinterpret_cast<float*>(Vs + B * P);
  float* s_vsum = s_kbar + D;
  float* s_red = s_vsum + D;

  const int M = L / B;
  const int j = blockIdx.x, bh = blockIdx.y;
  const size_t head = (size_t)bh * L * D;
  load_tile_async<B, D>(Ks, K + head + (size_t)j * B * D);
  load_tile_async<B, D>(Vs, V + head + (size_t)j * B * D);
  cp_async_wait_all();
  __syncthreads();
  const int nv = real_tokens<B>(key_valid, j, status);
  if (nv < B) {
    zero_padding<B, D>(Ks, Vs, nv);
    __syncthreads();
  }
  column_stats<B, D>(Ks, Vs, s_kbar, s_vsum, nv);
  float acc[Tiling<D>::MT][Tiling<D>::NT][4] = {};
  ktv_accumulate<B, D>(acc, Ks, Vs);
  __syncthreads();
  const float* hb = Hbar + (size_t)bh * D * D;
  float* hj = Hblk ? Hblk + ((size_t)bh * M + j) * D * D : nullptr;
  float sq = 0.f;
  for_each_acc<D>(acc, [&](float& x, int a, int c) {
    const float h = x - s_kbar[a] * s_vsum[c];
    if (hj) hj[a * D + c] = h;
    const float diff = h - hb[a * D + c];
    sq += diff * diff;
  });
  sq = warp_sum(sq);
  if (threadIdx.x % 32 == 0) s_red[threadIdx.x / 32] = sq;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) s += s_red[w];
    Mnorm[(size_t)bh * M + j] = sqrtf(s);
  }
}

// Blocks per k_pre_stats CTA: enough CTAs to cover the GPU a few times over while
// keeping the partial-sum scratch small.
int group_size(const Shape& s) {
  const long long blocks = (long long)s.BH() * s.M();
  int g = 1;
  while (g < 32 && blocks / g > 400) g *= 2;
  return g;
}

template <int B, int D>
size_t smem_bytes() {
  return 2 * (size_t)B * TilePitch<D>::elems * 2 + (2 * D + 32) * sizeof(float);
}

template <int B, int D>
cudaError_t run(const Shape& s, const void* K, const void* V, float* kbar, float* vsum,
                float* Hbar, float* Mnorm, float* Hblk, void* ws, int32_t* status,
                cudaStream_t st) {
  const int M = s.M(), G = group_size(s), n_grp = ceil_div(M, G);
  const size_t sm = smem_bytes<B, D>();
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(k_pre_stats<B, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)sm)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(k_pre_norm<B, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)sm)) != cudaSuccess)
    return e;
  float* partial = static_cast<float*>(ws);
  const auto* Kb = static_cast<const __nv_bfloat16*>(K);
  const auto* Vb = static_cast<const __nv_bfloat16*>(V);
  k_pre_stats<B, D><<<dim3(n_grp, s.BH()), kThreads, sm, st>>>(Kb, Vb, s.L, G, s.key_valid,
                                                               kbar, vsum, partial, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_pre_reduce<<<dim3(ceil_div(D * D, 256), s.BH()), 256, 0, st>>>(partial, n_grp, D * D, M,
                                                                   Hbar);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_pre_norm<B, D><<<dim3(M, s.BH()), kThreads, sm, st>>>(Kb, Vb, s.L, s.key_valid, Hbar,
                                                          Mnorm, Hblk, status);
  return cudaGetLastError();
}

}  // namespace

size_t precompute_workspace(const Shape& s) {
  if (s.d == 128) return precompute_tc_workspace(s);
  const int n_grp = ceil_div(s.M(), group_size(s));
  return (size_t)s.BH() * n_grp * s.d * s.d * sizeof(float);
}

cudaError_t launch_precompute(const Shape& s, const void* K, const void* V, float* kbar,
                              float* vsum, float* Hbar, float* Mnorm, float* Hblk, void* ws,
                              int32_t* status, cudaStream_t st) {
  // d = 128: tensor-core kernels (precompute_tc.cu); d = 64 (an M = 64 tcgen05 tile has a
  // different TMEM layout) keeps the mma.sync kernels of this file
  if (s.d == 128)
    return launch_precompute_tc(s, K, V, kbar, vsum, Hbar, Mnorm, Hblk, ws, status, st);
  if (s.block == 64) return run<64, 64>(s, K, V, kbar, vsum, Hbar, Mnorm, Hblk, ws, status, st);
  return run<128, 64>(s, K, V, kbar, vsum, Hbar, Mnorm, Hblk, ws, status, st);
}

}  // namespace bsa
