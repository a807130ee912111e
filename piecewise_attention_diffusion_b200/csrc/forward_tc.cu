// bsa_forward on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
// Method ("多模态 DiT 上的块稀疏 Attention" §3.3/§4.4; "PISA: Piecewise Sparse Attention
// Is Wiser for Efficient Diffusion Transformers", technical summary §2):
//   exact stage      for every selected KV block j in S_i: S = Q_i K_j^T, online softmax
//                    (running row max m, running denominator l), O += P V_j;
//   zeroth order     (PISA) the centroids kbar of the unselected blocks are swept in
//                    chunks of 128 as extra "key tiles": a = q . kbar_j, alpha = e^(a - m)
//                    with the same running max, O += alpha vsum_j, l += B alpha, and
//                    sum_alpha += alpha; selected and out-of-range centroids are masked;
//   first order      (PISA) T = Q Hbar on the tensor cores; the epilogue writes
//                    o = (O + s * sum_alpha * T) / l.
//
// Design (one persistent CTA per SM, 192 threads, warp-specialised):
//   warp 0  TMA producer: Q tiles (double-buffered) and a 4-slot ring of K / V /
//           centroid / Hbar tiles, each 128-byte swizzled, completion on mbarriers;
//   warp 1  MMA issuer (one thread): S = Q K^T into TMEM (two S buffers so the next
//           QK^T runs while the softmax works on the current one), O += P V with P read
//           from TMEM (bf16, aliased onto its own S buffer), T = Q Hbar;
//   warps 2-5  softmax: thread r owns query row r (TMEM lane r); loads its S row with
//           tcgen05.ld, applies the masks, exponentiates with ex2 in the log2 domain and
//           writes P back with tcgen05.st. O is rescaled in TMEM only when the running
//           max grows by more than 2^8 (the bound keeps every P <= 256, safe in bf16 and
//           fp32), so most tiles need no correction pass. The same warps run the
//           epilogue.
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D), T [256+D, 256+2D).
// Query tiles are 128 rows: one query block of 128, or two of 64 whose key-block lists
// are merged (each row masks the key blocks its own block does not select).
// Every mbarrier wait is bounded (sm100::mbar_wait); on a timeout the CTA drains its
// in-flight copies and MMAs, frees TMEM and reports BSA_ERR_TIMEOUT.
#include <limits.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace bsa {
namespace fwdtc {

using namespace sm100;

constexpr int kBQ = 128;       // query rows per tile
constexpr int kChunk = 128;    // centroids per sweep tile
constexpr int kThreads = 192;  // 6 warps
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

struct Params {
  int L, M, BH, n_qt, n_items;
  int qbox;  // rows per Q box: 128, or L when L < 128
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int csr_per_head;
  int pisa;
  float scale, scale_log2;
  __nv_bfloat16* O;
  float* lse;
  const int32_t* flag;
  int32_t* status;
};

template <int D, int BKV>
struct Cfg {
  static constexpr int QBPT = kBQ / BKV;          // query blocks per tile (1 or 2)
  static constexpr int QBYTES = kBQ * D * 2;
  static constexpr int SLOT = kBQ * D * 2;        // a slot holds up to 128 rows x D
  static constexpr int NSLOT = D == 128 ? 4 : 8;
  static constexpr int SMEM = 2 * QBYTES + NSLOT * SLOT + 1024;
  static constexpr uint32_t O_COL = 256u;
  static constexpr uint32_t T_COL = 256u + D;
};

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

template <int QBPT>
__device__ __forceinline__ Lists item_lists(const Params& p, int bh, int qt) {
  const int32_t* rp = p.csr_per_head ? p.row_ptr + (size_t)bh * (p.M + 1) : p.row_ptr;
  const int i0 = qt * QBPT;
  Lists r;
  r.col = p.col_idx;
  r.p0 = __ldg(rp + i0);
  r.e0 = __ldg(rp + i0 + 1);
  r.p1 = r.e1 = 0;
  if (QBPT == 2 && i0 + 1 < p.M) {
    r.p1 = r.e0;
    r.e1 = __ldg(rp + i0 + 2);
  }
  return r;
}

template <int QBPT>
__device__ __forceinline__ int count_exact(Lists l) {
  if (QBPT == 1) return l.e0 - l.p0;
  int n = 0;
  while (l.next() >= 0) ++n;
  return n;
}

struct Barriers {
  uint64_t q_full[2], q_empty[2];
  uint64_t kv_full[8], kv_empty[8];
  uint64_t s_full[2], p_full[2];
  uint64_t o_bar, o_final, o_free, done;
};

template <int D, int BKV>
__global__ void __launch_bounds__(kThreads, 1)
k_forward(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
          const __grid_constant__ CUtensorMap tmVs, const __grid_constant__ CUtensorMap tmHb,
          const Params p) {
  using C = Cfg<D, BKV>;
  if (*p.flag) return;  // malformed lists: leave O untouched

  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sSlot = smem + 2 * C::QBYTES;
  __shared__ Barriers bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.q_full[i], 1);
      mbar_init(&bars.q_empty[i], 1);
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.p_full[i], 128);
    }
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(&bars.kv_full[i], 1);
      mbar_init(&bars.kv_empty[i], 1);
    }
    mbar_init(&bars.o_bar, 1);
    mbar_init(&bars.o_final, 1);
    mbar_init(&bars.o_free, 128);
    mbar_init(&bars.done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    if (p.pisa) {
      prefetch_tensormap(&tmKb);
      prefetch_tensormap(&tmVs);
      prefetch_tensormap(&tmHb);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;
  const int n_ch = p.pisa ? ceil_div(p.M, kChunk) : 0;

  if (warp == 0) {
    // =============================================================== TMA producer
    if (lane == 0) {
      uint32_t ring = 0;
      int it = 0;
      int q_issued = 0;
      bool ok = true;
      auto load_slot = [&](int kind, int t_idx, int j, int bh) -> bool {
        // kind 0: K block j, 1: V block j, 2: centroid chunk, 3: value-sum chunk, 4: Hbar
        const int slot = ring % C::NSLOT;
        const uint32_t ph = (ring / C::NSLOT) & 1;
        if (!mbar_wait(&bars.kv_empty[slot], ph ^ 1, abort_flag)) return false;
        unsigned char* dst = sSlot + slot * C::SLOT;
        const int rows = kind <= 1 ? BKV : (kind == 4 ? D : kChunk);
        mbar_arrive_expect_tx(&bars.kv_full[slot], rows * D * 2);
        const CUtensorMap* map = kind == 0 ? &tmK : kind == 1 ? &tmV : kind == 2 ? &tmKb
                                 : kind == 3 ? &tmVs : &tmHb;
        const int y = kind <= 1 ? j * BKV : (kind == 4 ? 0 : j * kChunk);
        // one 4-D box: 64 columns x rows x (D/64) column groups; lands as D/64 swizzled
        // [rows x 64] sub-tiles, sub-tile h at byte offset h * rows * 128
        tma_load_4d(dst, map, &bars.kv_full[slot], 0, y, 0, bh);
        ++ring;
        (void)t_idx;
        return true;
      };
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++it) {
        const int bh = item / p.n_qt, qt = item % p.n_qt;
        const Lists lists = item_lists<C::QBPT>(p, bh, qt);
        const int n_ex = count_exact<C::QBPT>(lists);
        const int n = n_ex + n_ch;
        const int qb = it & 1;
        if (!mbar_wait(&bars.q_empty[qb], ((it >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars.q_full[qb], p.qbox * D * 2);
        if (p.qbox == kBQ) {
          tma_load_4d(smem + qb * C::QBYTES, &tmQ, &bars.q_full[qb], 0, qt * kBQ, 0, bh);
        } else {  // L < 128: one box per column group, at the 128-row sub-tile stride
#pragma unroll
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(smem + qb * C::QBYTES + h * kBQ * 128, &tmQ, &bars.q_full[qb], 0, 0, h, bh);
        }
        ++q_issued;
        Lists lk = lists, lv = lists;
        for (int t = 0; t < n && ok; ++t) {
          if (t < n_ex) ok = load_slot(0, t, lk.next(), bh);
          else ok = load_slot(2, t, t - n_ex, bh);
          if (ok && t >= 1) {
            const int u = t - 1;
            if (u < n_ex) ok = load_slot(1, u, lv.next(), bh);
            else ok = load_slot(3, u, u - n_ex, bh);
          }
        }
        if (ok && n >= 1) {
          const int u = n - 1;
          if (u < n_ex) ok = load_slot(1, u, lv.next(), bh);
          else ok = load_slot(3, u, u - n_ex, bh);
        }
        if (ok && p.pisa) ok = load_slot(4, 0, 0, bh);
      }
      if (!ok) {
        // drain: wait (bounded, ignoring the abort flag) for copies still in flight
        const uint64_t t0 = globaltimer_ns();
        const uint32_t first = ring > (uint32_t)C::NSLOT ? ring - C::NSLOT : 0;
        for (uint32_t r = first; r < ring; ++r) {
          while (!mbar_try_wait(&bars.kv_full[r % C::NSLOT], (r / C::NSLOT) & 1) &&
                 globaltimer_ns() - t0 < 100000000ull) {
          }
        }
        for (int r = max(0, q_issued - 2); r < q_issued; ++r) {
          while (!mbar_try_wait(&bars.q_full[r & 1], (r >> 1) & 1) &&
                 globaltimer_ns() - t0 < 100000000ull) {
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      uint32_t ring = 0, g = 0;
      int it = 0;
      bool ok = true;
      constexpr uint32_t idesc_s_ex = idesc_bf16_f32(kBQ, BKV, false, false);
      constexpr uint32_t idesc_s_ch = idesc_bf16_f32(kBQ, kChunk, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kBQ, D, false, true);
      auto wait_slot = [&](uint32_t& slot_out) -> bool {
        const int slot = ring % C::NSLOT;
        if (!mbar_wait(&bars.kv_full[slot], (ring / C::NSLOT) & 1, abort_flag)) return false;
        tc_fence_after();
        slot_out = slot;
        ++ring;
        return true;
      };
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++it) {
        const int bh = item / p.n_qt, qt = item % p.n_qt;
        const Lists lists = item_lists<C::QBPT>(p, bh, qt);
        const int n_ex = count_exact<C::QBPT>(lists);
        const int n = n_ex + n_ch;
        const int qb = it & 1;
        if (!mbar_wait(&bars.q_full[qb], (it >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t q_addr = smem_u32(smem + qb * C::QBYTES);
        bool o_free_done = (it == 0);
        auto wait_o_free = [&]() -> bool {
          if (o_free_done) return true;
          if (!mbar_wait(&bars.o_free, (it - 1) & 1, abort_flag)) return false;
          tc_fence_after();
          o_free_done = true;
          return true;
        };
        auto issue_pv = [&](int u) -> bool {
          const uint32_t gu = g + u, buf = gu & 1;
          if (!mbar_wait(&bars.p_full[buf], (gu >> 1) & 1, abort_flag)) return false;
          tc_fence_after();
          uint32_t slot;
          if (!wait_slot(slot)) return false;
          if (u == 0 && !wait_o_free()) return false;
          const bool chunk = u >= n_ex;
          const int kdim = chunk ? kChunk : BKV;
          const uint32_t v_addr = smem_u32(sSlot + slot * C::SLOT);
          for (int k = 0; k < kdim / 16; ++k) {
            const uint64_t bdesc = smem_desc_sw128(v_addr + k * 2048, kdim * 128, 1024);
            mma_ts(tmem + C::O_COL, tmem + (buf ? 128u : 0u) + k * 8, bdesc, idesc_o,
                   (u > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(&bars.kv_empty[slot]);
          mma_commit(&bars.o_bar);
          return true;
        };
        for (int t = 0; t < n && ok; ++t) {
          uint32_t slot;
          if (!wait_slot(slot)) { ok = false; break; }
          const bool chunk = t >= n_ex;
          const int rows = chunk ? kChunk : BKV;
          const uint32_t buf = (g + t) & 1;
          const uint32_t k_addr = smem_u32(sSlot + slot * C::SLOT);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint64_t adesc =
                smem_desc_sw128(q_addr + (k / 4) * (kBQ * 128) + (k % 4) * 32, 16, 1024);
            const uint64_t bdesc =
                smem_desc_sw128(k_addr + (k / 4) * (rows * 128) + (k % 4) * 32, 16, 1024);
            mma_ss(tmem + (buf ? 128u : 0u), adesc, bdesc, chunk ? idesc_s_ch : idesc_s_ex,
                   k > 0 ? 1u : 0u);
          }
          mma_commit(&bars.kv_empty[slot]);
          mma_commit(&bars.s_full[buf]);
          if (t >= 1 && !issue_pv(t - 1)) { ok = false; break; }
        }
        if (ok && n >= 1) ok = issue_pv(n - 1);
        if (ok && p.pisa) {
          uint32_t slot;
          ok = wait_slot(slot) && wait_o_free();
          if (ok) {
            const uint32_t h_addr = smem_u32(sSlot + slot * C::SLOT);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint64_t adesc =
                  smem_desc_sw128(q_addr + (k / 4) * (kBQ * 128) + (k % 4) * 32, 16, 1024);
              const uint64_t bdesc = smem_desc_sw128(h_addr + k * 2048, D * 128, 1024);
              mma_ss(tmem + C::T_COL, adesc, bdesc, idesc_o, k > 0 ? 1u : 0u);
            }
            mma_commit(&bars.kv_empty[slot]);
          }
        }
        if (ok) ok = wait_o_free();
        if (!ok) break;
        mma_commit(&bars.q_empty[qb]);
        mma_commit(&bars.o_final);
        g += n;
      }
      // every issued MMA must complete before TMEM is released
      mma_commit(&bars.done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&bars.done, 0) && globaltimer_ns() - t0 < 100000000ull) {
      }
    }
    __syncwarp();
  } else {
    // ============================================================ softmax + epilogue
    const int quad = warp % 4;                 // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;          // query row within the tile
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    uint32_t g = 0, pv = 0;
    int it = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++it) {
      const int bh = item / p.n_qt, qt = item % p.n_qt;
      Lists lists = item_lists<C::QBPT>(p, bh, qt);
      const int n_ex = count_exact<C::QBPT>(lists);
      const int n = n_ex + n_ch;
      const int row_g = qt * kBQ + row;
      const int iq = qt * C::QBPT + row / BKV;   // this row's query block
      const bool has_blk = iq < p.M;
      const int32_t* rp = p.csr_per_head ? p.row_ptr + (size_t)bh * (p.M + 1) : p.row_ptr;
      const int mb = has_blk ? __ldg(rp + iq) : 0;
      const int me = has_blk ? __ldg(rp + iq + 1) : 0;
      int mp = mb, cp = mb;
      float m_run = -INFINITY, l = 0.f, sa = 0.f;

      for (int t = 0; t < n; ++t) {
        const uint32_t gt = g + t, buf = gt & 1;
        ok = mbar_wait(&bars.s_full[buf], (gt >> 1) & 1, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const bool chunk = t >= n_ex;
        const uint32_t s_addr = tmem + lane_addr + (buf ? 128u : 0u);
        float s[128];
        {
          uint32_t r[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (c * 32 < (chunk ? kChunk : BKV)) {
              tmem_ld32(s_addr + c * 32, r);
#pragma unroll
              for (int x = 0; x < 32; ++x) s[c * 32 + x] = __uint_as_float(r[x]);
            }
          }
          tmem_wait_ld();
        }
        // tile width: 128 for centroid chunks, BKV for exact tiles (compile-time for 128)
        const int N = BKV == kChunk ? kChunk : (chunk ? kChunk : BKV);
        if (!chunk) {
          if (C::QBPT == 2) {
            const int j = lists.next();
            const bool member = mp < me && __ldg(p.col_idx + mp) == j;
            if (member) ++mp;
            if (!member) {
#pragma unroll
              for (int x = 0; x < BKV; ++x) s[x] = -INFINITY;
            }
          }
        } else {
          // centroid chunk: mask selected blocks and indices past M
          const int base = (t - n_ex) * kChunk;
          uint32_t excl[4] = {0u, 0u, 0u, 0u};
          while (cp < me) {
            const int cj = __ldg(p.col_idx + cp);
            if (cj >= base + kChunk) break;
            if (cj >= base) excl[(cj - base) >> 5] |= 1u << ((cj - base) & 31);
            ++cp;
          }
          const int valid = has_blk ? min(kChunk, p.M - base) : 0;
#pragma unroll
          for (int x = 0; x < kChunk; ++x)
            if (x >= valid || ((excl[x >> 5] >> (x & 31)) & 1u)) s[x] = -INFINITY;
        }
        // row max (log2 domain); 8 independent chains keep the FMNMX latency hidden
        float mxa[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) mxa[a] = s[a];
#pragma unroll
        for (int x = 8; x < 128; x += 8) {
          if (x < N) {
#pragma unroll
            for (int a = 0; a < 8; ++a) mxa[a] = fmaxf(mxa[a], s[x + a]);
          }
        }
        const float mx = fmaxf(fmaxf(fmaxf(mxa[0], mxa[1]), fmaxf(mxa[2], mxa[3])),
                               fmaxf(fmaxf(mxa[4], mxa[5]), fmaxf(mxa[6], mxa[7]))) *
                         p.scale_log2;
        const bool need = mx > m_run + kRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          const float m_new = need ? mx : m_run;
          const float factor = need ? ex2(m_run - m_new) : 1.0f;
          if (t > 0) {
            ok = mbar_wait(&bars.o_bar, (pv + t - 1) & 1, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const uint32_t o_addr = tmem + lane_addr + C::O_COL;
#pragma unroll 1
            for (int c = 0; c < D; c += 32) {
              uint32_t r[32];
              tmem_ld32(o_addr + c, r);
              tmem_wait_ld();
#pragma unroll
              for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * factor);
              tmem_st32(o_addr + c, r);
            }
            tmem_wait_st();
          }
          l *= factor;
          sa *= factor;
          m_run = m_new;
        }
        const float m_ref = m_run == -INFINITY ? 0.f : m_run;
        // P = 2^(s*scale_log2 - m) as bf16 pairs, written back over the first N/2
        // columns of this S buffer one 64-column half at a time (all S values are
        // already in registers, so the overwrite is safe)
        const uint32_t p_addr = tmem + lane_addr + (buf ? 128u : 0u);
        float sm[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          if (hf * 64 < N) {
            uint32_t pk[32];
#pragma unroll
            for (int x = 0; x < 64; x += 2) {
              const float e0 = ex2(fmaf(s[hf * 64 + x], p.scale_log2, -m_ref));
              const float e1 = ex2(fmaf(s[hf * 64 + x + 1], p.scale_log2, -m_ref));
              sm[(x / 2) & 7] += e0 + e1;
              pk[x / 2] = pack_bf16x2(e0, e1);
            }
            tmem_st32(p_addr + hf * 32, pk);
          }
        }
        const float rs = ((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7]));
        if (chunk) {
          l += (float)BKV * rs;
          sa += rs;
        } else {
          l += rs;
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars.p_full[buf]);
      }
      if (!ok) break;

      // ---------------------------------------------------------------- epilogue
      ok = mbar_wait(&bars.o_final, it & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const bool write = row_g < p.L;
      __nv_bfloat16* orow = p.O + ((size_t)bh * p.L + (write ? row_g : 0)) * D;
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      const float c1 = p.scale * sa;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t ro[32], rt[32];
        if (n > 0) {
          tmem_ld32(tmem + lane_addr + C::O_COL + c, ro);
          if (p.pisa) tmem_ld32(tmem + lane_addr + C::T_COL + c, rt);
          tmem_wait_ld();
        }
        uint32_t packed[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          float a0 = 0.f, a1 = 0.f;
          if (n > 0) {
            a0 = __uint_as_float(ro[x]);
            a1 = __uint_as_float(ro[x + 1]);
            if (p.pisa) {
              a0 = fmaf(c1, __uint_as_float(rt[x]), a0);
              a1 = fmaf(c1, __uint_as_float(rt[x + 1]), a1);
            }
          }
          packed[x / 2] = pack_bf16x2(a0 * inv_l, a1 * inv_l);
        }
        if (write) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2],
                                packed[4 * v + 3]);
        }
      }
      if (write && p.lse)
        p.lse[(size_t)bh * p.L + row_g] =
            l > 0.f ? (m_run + log2f(l)) * 0.69314718055994531f : -INFINITY;
      tc_fence_before();
      mbar_arrive(&bars.o_free);
      g += n;
      pv += n;
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

// Convert the PISA statistics to bf16 operands. kbar and vsum [BH, M, D] become
// [BH, Mp, D] with Mp = M rounded up to a multiple of 128 (pad rows zero, so every
// centroid tile is a full in-bounds TMA box); Hbar [BH, D, D] is converted as is.
__global__ void k_stats_bf16(const float4* __restrict__ kbar, const float4* __restrict__ vsum,
                             const float4* __restrict__ Hbar, uint2* __restrict__ kb16,
                             uint2* __restrict__ vs16, uint2* __restrict__ hb16, int M, int Mp,
                             int D4, size_t n_kv4, size_t n_h4) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_kv4 + n_h4; i += stride) {
    if (i < n_kv4) {
      const size_t row = i / D4, c4 = i % D4;
      const size_t bh = row / Mp, m = row % Mp;
      if ((int)m < M) {
        const size_t src = (bh * M + m) * D4 + c4;
        const float4 a = kbar[src], b = vsum[src];
        kb16[i] = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
        vs16[i] = make_uint2(pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
      } else {
        kb16[i] = make_uint2(0u, 0u);
        vs16[i] = make_uint2(0u, 0u);
      }
    } else {
      const float4 h = Hbar[i - n_kv4];
      hb16[i - n_kv4] = make_uint2(pack_bf16x2(h.x, h.y), pack_bf16x2(h.z, h.w));
    }
  }
}

// ------------------------------------------------------------------ host side
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

// bf16 tensor [z][rows][cols] (cols contiguous, cols a multiple of 64) viewed as 4-D
// (64 columns, rows, cols/64 column groups, z) so that one box of 64 x box_rows x
// cols/64 lands in shared memory as cols/64 consecutive [box_rows x 64] sub-tiles, each
// 128-byte swizzled: the operand layout of the MMA descriptors (sub-tile h at byte
// offset h * box_rows * 128). With all_groups false the box holds one column group, for
// callers that place the groups themselves (a Q tile shorter than 128 rows).
bool make_map(CUtensorMap* m, const void* ptr, int cols, int rows, int z, int box_rows,
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

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int D, int BKV>
cudaError_t run(const ForwardArgs& a, const int32_t* flag, const void* kb16, const void* vs16,
                const void* hb16, cudaStream_t st) {
  using C = Cfg<D, BKV>;
  const Shape& s = a.s;
  const int BH = s.BH(), M = s.M();
  CUtensorMap tmQ, tmK, tmV, tmKb, tmVs, tmHb;
  const int qbox = s.L < kBQ ? s.L : kBQ;
  const int Mp = ceil_div(M, kChunk) * kChunk;
  bool ok = make_map(&tmQ, a.Q, D, s.L, BH, qbox, qbox == kBQ) &&
            make_map(&tmK, a.K, D, s.L, BH, BKV) &&
            make_map(&tmV, a.V, D, s.L, BH, BKV);
  if (a.mode == BSA_MODE_PISA) {
    ok = ok && make_map(&tmKb, kb16, D, Mp, BH, kChunk) && make_map(&tmVs, vs16, D, Mp, BH, kChunk) &&
         make_map(&tmHb, hb16, D, D, BH, D);
  } else {
    tmKb = tmVs = tmHb = tmK;  // unused
  }
  if (!ok) return cudaErrorInvalidValue;
  Params p;
  p.L = s.L;
  p.M = M;
  p.BH = BH;
  p.n_qt = ceil_div(s.L, kBQ);
  p.n_items = BH * p.n_qt;
  p.qbox = qbox;
  p.row_ptr = a.row_ptr;
  p.col_idx = a.col_idx;
  p.csr_per_head = a.csr_per_head;
  p.pisa = a.mode == BSA_MODE_PISA;
  p.scale = a.scale;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.O = static_cast<__nv_bfloat16*>(a.O);
  p.lse = a.lse;
  p.flag = flag;
  p.status = a.status;
  cudaError_t e = cudaFuncSetAttribute(k_forward<D, BKV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int grid = min(p.n_items, sm_count());
  k_forward<D, BKV><<<grid, kThreads, C::SMEM, st>>>(tmQ, tmK, tmV, tmKb, tmVs, tmHb, p);
  return cudaGetLastError();
}

}  // namespace fwdtc

// Workspace: [0,256) flag; then bf16 kbar, vsum [BH, Mp, D] (Mp = M rounded up to 128)
// and Hbar [BH, D, D].
namespace {
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
size_t padded_blocks(const Shape& s) { return (size_t)ceil_div(s.M(), fwdtc::kChunk) * fwdtc::kChunk; }
}  // namespace

size_t forward_tc_workspace(const Shape& s) {
  const size_t kv = (size_t)s.BH() * padded_blocks(s) * s.d * 2;
  const size_t h = (size_t)s.BH() * s.d * s.d * 2;
  return 256 + 2 * align256(kv) + align256(h);
}

cudaError_t launch_forward_tc(const ForwardArgs& a, const int32_t* flag, cudaStream_t st) {
  const Shape& s = a.s;
  unsigned char* ws = static_cast<unsigned char*>(a.ws);
  const size_t Mp = padded_blocks(s);
  const size_t kv = align256((size_t)s.BH() * Mp * s.d * 2);
  void* kb16 = ws + 256;
  void* vs16 = ws + 256 + kv;
  void* hb16 = ws + 256 + 2 * kv;
  if (a.mode == BSA_MODE_PISA) {
    const size_t n_kv4 = (size_t)s.BH() * Mp * s.d / 4, n_h4 = (size_t)s.BH() * s.d * s.d / 4;
    const int blocks = (int)std::min<size_t>((n_kv4 + n_h4 + 255) / 256, 4096);
    fwdtc::k_stats_bf16<<<blocks, 256, 0, st>>>(
        reinterpret_cast<const float4*>(a.kbar), reinterpret_cast<const float4*>(a.vsum),
        reinterpret_cast<const float4*>(a.Hbar), static_cast<uint2*>(kb16),
        static_cast<uint2*>(vs16), static_cast<uint2*>(hb16), s.M(), (int)Mp, s.d / 4, n_kv4,
        n_h4);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (s.d == 64 && s.block == 64) return fwdtc::run<64, 64>(a, flag, kb16, vs16, hb16, st);
  if (s.d == 64 && s.block == 128) return fwdtc::run<64, 128>(a, flag, kb16, vs16, hb16, st);
  if (s.d == 128 && s.block == 64) return fwdtc::run<128, 64>(a, flag, kb16, vs16, hb16, st);
  return fwdtc::run<128, 128>(a, flag, kb16, vs16, hb16, st);
}

}  // namespace bsa
