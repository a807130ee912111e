// bsa_forward in the keep-or-drop and PISA modes on the 5th-generation tensor cores
// (tcgen05 + TMEM + TMA), sm_100a: every query row's softmax is shared by a pair of
// threads, one per half of the score row. Used at head dim 64, where it measured faster
// than the kernel with one thread per row (forward_tc.cu); at head dim 128 that kernel is
// the faster one, since here every exponential also pays for the rounded row sum below.
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
// Why pairs. Each of the two query tiles in flight ("streams") runs softmax(t) -> PV(t),
// S(t+1) -> softmax(t+1) in series: tensor memory (512 columns) holds per stream one
// 128-column score tile and its O accumulator, so the next scores cannot be computed
// while P still occupies the score tile. The tensor core is therefore busy only while
// the other stream's softmax runs, and the length of one softmax bounds the whole kernel.
// Two warpgroups per stream, each owning 64 of the 128 score columns, halve it; they
// agree on the row maximum through shared memory before exponentiating.
//
// Design (one persistent CTA per SM, 576 threads, warp-specialised):
//   warps 0-3 / 4-7    stream 0, column halves 0 / 1; warps 8-11 / 12-15: stream 1.
//           Thread r of a half owns query row r (TMEM lane r). Per tile: its half of the
//           S row into registers, the half's row max, the pair's max (bf16 in shared
//           memory, a named barrier of the stream's 256 threads that also agrees on
//           aborting), the lazy rescale of its half of O when the running max grows by
//           more than 2^8, P = 2^(s*scale*log2(e) - m) with a quarter of the exponentials
//           on the FMA pipe, stored as bf16 pairs at the start of the half's own score
//           columns (so the halves never write over each other's scores; the MMA issuer
//           takes each K-step's P from the half that holds its keys). The same warps run
//           the epilogue (each half writes its half of O's columns) and load the stream's
//           query tiles.
//   warp 16  TMA producer of a ring of K / V / centroid / value-sum / Hbar tiles,
//           in the MMA issuer's step order, both streams alternating;
//   warp 17  MMA issuer (one thread): per stream step, O += P(t-1) V(t-1) (P is the
//           TMEM A operand) then S(t) = Q K(t)^T; last step of an item T = Q Hbar into
//           the freed score tile.
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256, 256+D), O1 [256+D, 256+2D).
// Query tiles are 128 rows: one query block of 128, or two of 64 whose key-block lists
// are merged (each row masks the key blocks its own block does not select). With
// 64-token blocks (and L >= 128) the exact steps are pairs of key blocks, 128 keys wide:
// each half of a row owns one block of the pair and skips it when the row's own list
// lacks it (see Steps).
// Every mbarrier wait is bounded (sm100::mbar_wait); on a timeout the CTA drains its
// in-flight copies and MMAs, frees TMEM and reports BSA_ERR_TIMEOUT.
#include <limits.h>

#include <algorithm>

#include "common.cuh"
#include "forward_tiles.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace bsa {
namespace fwdpair {

using namespace sm100;
using namespace fwdtiles;

constexpr int kBQ = 128;       // query rows per tile
constexpr int kChunk = 128;    // centroids per sweep tile
constexpr int kStreams = 2;    // query tiles in flight per CTA
constexpr int kHalves = 2;     // softmax warpgroups per stream
constexpr int kSoftmaxWarps = 4 * kStreams * kHalves;
constexpr int kThreads = 32 * kSoftmaxWarps + 64;   // softmax warpgroups, producer, MMA issuer
constexpr int kProducerWarp = kSoftmaxWarps;
constexpr int kMmaWarp = kProducerWarp + 1;
// 576 threads, one CTA per SM: 96 registers per thread. The register file is split over the
// SM's four schedulers and two of them hold five of the 18 warps: 16384 / (5 * 32) rounded
// down to a multiple of 8. That holds a half score row (64 values) and its packed P.
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t kAll = 0xffffffffu;

struct Params {
  int L, M, BH, n_qt, n_items;
  int tile_major;  // items ordered (tile, head) instead of (head, tile): lists shared by all heads
  int qbox;  // rows per Q box: 128, or L when L < 128
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int csr_per_head;
  int pisa;
  const int32_t* key_valid;  // real tokens per block, or null (no padding)
  float scale, scale_log2;
  __nv_bfloat16* O;
  float* lse;
  const int32_t* flag;
  int32_t* status;
  uint64_t wait_ns;  // limit of every bounded wait
};

// Head and query tile of work item `item`. With one list shared by every head (a fixed
// mask) the items go tile by tile, every head's tile qt before any head's tile qt + 1, so
// that the first items dealt are the heads' first tiles (in the multimodal layout the
// text rows, whose lists are the longest); with per-head lists, head by head (a head's
// K and V stay in L2 while its tiles run).
__device__ __forceinline__ void item_tile(const Params& p, int item, int& bh, int& qt) {
  if (p.tile_major) {
    qt = item / p.BH;
    bh = item % p.BH;
  } else {
    bh = item / p.n_qt;
    qt = item % p.n_qt;
  }
}

template <int D, int BKV, bool KP>
struct Cfg {
  static constexpr int QBPT = kBQ / BKV;          // query blocks per tile (1 or 2)
  static constexpr int KT = KP ? 2 * BKV : BKV;   // keys per exact step
  static constexpr int QBYTES = kBQ * D * 2;
  static constexpr int SLOT = kBQ * D * 2;        // a slot holds up to 128 rows x D
  static constexpr int NSLOT = D == 128 ? 5 : 8;
  static constexpr int SMEM = kStreams * QBYTES + NSLOT * SLOT + 1024;
  static constexpr int HALF_EX = KT / 2;          // columns of a half of an exact tile
  static constexpr int HALF_D = D / 2;            // columns of a half of O
  __host__ __device__ static constexpr uint32_t S_COL(int x) { return 128u * x; }
  __host__ __device__ static constexpr uint32_t O_COL(int x) { return 256u + D * x; }
};

struct Barriers {
  uint64_t kv_full[8], kv_empty[8];
  uint64_t q_full[kStreams];
  uint64_t s_full[kStreams], p_full[kStreams];
  uint64_t o_final[kStreams], o_free[kStreams], o_staged[kStreams];
  uint64_t done;
};

// Work item k of stream x of this CTA (static schedule: the CTA takes items
// blockIdx.x, blockIdx.x + G, ... and deals them to its two streams alternately).
__device__ __forceinline__ int stream_item(int k, int x) {
  return blockIdx.x + (2 * k + x) * gridDim.x;
}

// The exact steps of a tile. Without KP a step is one key block j of its lists (merged);
// with KP (64-token blocks, paired) a step is a pair m of key blocks 2m and 2m + 1, taken
// once if the lists hold either, so that every step is a 128-key tile: the two softmax
// halves of a row each own one block, and a row skips a half whose block is not in its
// own list.
template <bool KP>
struct Steps {
  Lists l;
  int pend;  // with KP: the lists' next key block (-1 at the end)
  __device__ __forceinline__ void init(const Lists& x) {
    l = x;
    if (KP) pend = l.next();
  }
  __device__ __forceinline__ int next() {
    if (!KP) return l.next();
    if (pend < 0) return -1;
    const int m = pend >> 1;
    pend = l.next();
    if (pend >= 0 && (pend >> 1) == m) pend = l.next();
    return m;
  }
};

template <bool KP, int QBPT>
__device__ __forceinline__ int count_steps(const Lists& l) {
  if (!KP) return count_exact<QBPT>(l);
  Steps<true> st;
  st.init(l);
  int n = 0;
  while (st.next() >= 0) ++n;
  return n;
}

// Per-stream position in the step schedule shared by the producer and the MMA issuer.
// Steps of an item with n tiles: step 0 = S(0); step t (1 <= t < n) = PV(t-1), S(t);
// step n = PV(n-1) [+ T] and the end of the item. An item with n = 0 has one step.
template <int QBPT, bool KP>
struct StreamPos {
  int k, item, bh, qt, n, n_ex, t;
  uint32_t tiles;  // tiles of earlier items of this stream (barrier phases)
  int items;       // earlier items of this stream
  Steps<KP> lk, lv;  // K-side and V-side step cursors (producer)
  __device__ __forceinline__ void start(const Params& p, int x, int n_ch) {
    item = stream_item(k, x);
    if (item >= p.n_items) return;
    item_tile(p, item, bh, qt);
    const Lists li = item_lists<QBPT>(p.row_ptr, p.col_idx, p.csr_per_head, p.M, bh, qt);
    lk.init(li);
    lv = lk;
    n_ex = count_steps<KP, QBPT>(li);
    n = n_ex + n_ch;
    t = 0;
  }
  __device__ __forceinline__ bool active(const Params& p) const { return item < p.n_items; }
  __device__ __forceinline__ void advance(const Params& p, int x, int n_ch) {
    tiles += n;
    ++items;
    ++k;
    start(p, x, n_ch);
  }
};

enum LoadKind { kLoadK = 0, kLoadV = 1, kLoadKbar = 2, kLoadVsum = 3, kLoadHbar = 4 };

__device__ __forceinline__ void bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Exclusion bits (2 words) of the columns [v, 64) of a half tile.
__device__ __forceinline__ void tail_bits(int v, uint32_t& w0, uint32_t& w1) {
  w0 = v <= 0 ? kAll : (v < 32 ? kAll << v : 0u);
  w1 = v <= 32 ? kAll : (v < 64 ? kAll << (v - 32) : 0u);
}

// P for N (= 32) columns held in r: 2^(s * scale_log2 - m_ref), stored to TMEM as bf16
// pairs (column c holds elements 2c, 2c + 1) at p_addr, 8 columns at a time. Returns two
// sums: of the stored bf16 values (x), which normalise the output, so that every output
// is a weighted mean of value rows with the same weights in numerator and denominator;
// and of the fp32 values (y), for the log-sum-exp. With kMixed, kPolyOf8 of every 8 pairs
// run on the FMA pipe; with kMasked (a tile with excluded columns, -inf in r) those give
// exactly 0 for an excluded column, as the special-function unit does.
template <int N, bool kMixed, bool kMasked>
__device__ __forceinline__ float2 half_exp(const uint32_t (&r)[32], float scale_log2, float m_ref,
                                           uint32_t p_addr) {
  const float2 sc = make_float2(scale_log2, scale_log2);
  const float2 nm = make_float2(-m_ref, -m_ref);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f), acce = make_float2(0.f, 0.f);
#pragma unroll
  for (int h = 0; h < N / 16; ++h) {
    uint32_t pk[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = h * 16 + 2 * q;
      const float2 xx =
          fma2(make_float2(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), sc, nm);
      float2 ev;
      if (kMixed && q < kPolyOf8) {
        ev = ex2_poly2(xx);
        if (kMasked) {
          // the polynomial clamps its argument at -126: a masked score (-inf) must give 0
          ev.x = xx.x == -INFINITY ? 0.f : ev.x;
          ev.y = xx.y == -INFINITY ? 0.f : ev.y;
        }
      } else {
        ev = make_float2(ex2(xx.x), ex2(xx.y));
      }
      acce = add2(acce, ev);
      pk[q] = pack_bf16x2(ev.x, ev.y);
      // the bf16 values the PV MMA multiplies (the high half of each word is one bf16,
      // exactly an fp32 with zero low bits)
      const float2 pr = make_float2(__uint_as_float(pk[q] << 16), __uint_as_float(pk[q] & 0xffff0000u));
      if (q & 1) acc1 = add2(acc1, pr);
      else acc0 = add2(acc0, pr);
    }
    tmem_st8(p_addr + h * 8, pk);
  }
  const float2 a = add2(acc0, acc1);
  return make_float2(a.x + a.y, acce.x + acce.y);
}

// bf16 bits of x rounded towards +inf: the pair's shared row max. Both halves use the
// rounded values of both, so they agree exactly on the reference, and rounding up keeps
// the reference at or above the true maximum (every P <= 1 before the lazy rescale's
// allowance of 2^8).
__device__ __forceinline__ uint16_t bf16_bits(float x) {
  const __nv_bfloat16 b = __float2bfloat16_ru(x);
  return *reinterpret_cast<const uint16_t*>(&b);
}
__device__ __forceinline__ float bf16_value(uint16_t u) {
  return __uint_as_float((uint32_t)u << 16);
}

template <int D, int BKV, bool KP>
__global__ void __launch_bounds__(kThreads, 1)
k_pair(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
       const __grid_constant__ CUtensorMap tmVs, const __grid_constant__ CUtensorMap tmHb,
       const __grid_constant__ CUtensorMap tmO, const Params p) {
  using C = Cfg<D, BKV, KP>;
  if (*p.flag) return;  // malformed lists: leave O untouched

  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sSlot = smem + kStreams * C::QBYTES;
  __shared__ Barriers bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ uint16_t s_max[kStreams][kHalves][kBQ];  // each half's row max (bf16 bits)

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int x = 0; x < kStreams; ++x) {
      mbar_init(&bars.q_full[x], 1);
      mbar_init(&bars.s_full[x], 1);
      mbar_init(&bars.p_full[x], 128 * kHalves);
      mbar_init(&bars.o_final[x], 1);
      mbar_init(&bars.o_free[x], 128 * kHalves);
      mbar_init(&bars.o_staged[x], 128 * kHalves);
    }
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(&bars.kv_full[i], 1);
      mbar_init(&bars.kv_empty[i], 1);
    }
    mbar_init(&bars.done, 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
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
  if (warp == kProducerWarp) {
    // ================================================= TMA producer of the K/V ring
    if (lane == 0) {
      uint32_t ring = 0;
      bool ok = true;
      auto load = [&](int kind, int j, int bh) -> bool {
        const int slot = ring % C::NSLOT;
        const uint32_t ph = (ring / C::NSLOT) & 1;
        if (!mbar_wait(&bars.kv_empty[slot], ph ^ 1, abort_flag, p.wait_ns)) return false;
        unsigned char* dst = sSlot + slot * C::SLOT;
        const CUtensorMap* map = kind == kLoadK ? &tmK : kind == kLoadV ? &tmV
                                 : kind == kLoadKbar ? &tmKb : kind == kLoadVsum ? &tmVs : &tmHb;
        const int rows = kind <= kLoadV ? C::KT : (kind == kLoadHbar ? D : kChunk);
        const int y = kind <= kLoadV ? j * C::KT : (kind == kLoadHbar ? 0 : j * kChunk);
        mbar_arrive_expect_tx(&bars.kv_full[slot], rows * D * 2);
        // one 4-D box: 64 columns x rows x (D/64) column groups; lands as D/64 swizzled
        // [rows x 64] sub-tiles, sub-tile h at byte offset h * rows * 128
        tma_load_4d(dst, map, &bars.kv_full[slot], 0, y, 0, bh);
        ++ring;
        return true;
      };
      // the loads of one step of stream x, in the MMA issuer's order
      auto step = [&](StreamPos<C::QBPT, KP>& s, int x) -> bool {
        if (s.t == 0) {
          if (s.n == 0) {
            s.advance(p, x, n_ch);
            return true;
          }
          const bool r = s.n_ex > 0 ? load(kLoadK, s.lk.next(), s.bh) : load(kLoadKbar, 0, s.bh);
          s.t = 1;
          return r;
        }
        const int u = s.t - 1;
        if (!(u < s.n_ex ? load(kLoadV, s.lv.next(), s.bh) : load(kLoadVsum, u - s.n_ex, s.bh)))
          return false;
        if (s.t < s.n) {
          const bool r = s.t < s.n_ex ? load(kLoadK, s.lk.next(), s.bh)
                                      : load(kLoadKbar, s.t - s.n_ex, s.bh);
          ++s.t;
          return r;
        }
        const bool r = p.pisa ? load(kLoadHbar, 0, s.bh) : true;
        s.advance(p, x, n_ch);
        return r;
      };
      StreamPos<C::QBPT, KP> s0, s1;
      s0.k = s1.k = 0;
      s0.tiles = s1.tiles = 0;
      s0.items = s1.items = 0;
      s0.start(p, 0, n_ch);
      s1.start(p, 1, n_ch);
      while (ok && (s0.active(p) || s1.active(p))) {
        if (s0.active(p) && !(ok = step(s0, 0))) break;
        if (s1.active(p) && !(ok = step(s1, 1))) break;
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
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      // ring position as (slot, phase), advanced without division; `last` is the slot
      // of the most recent wait_slot
      uint32_t slot = 0, phase = 0, last = 0;
      bool ok = true;
      constexpr uint32_t idesc_s_ex = idesc_bf16_f32(kBQ, C::KT, false, false);
      constexpr uint32_t idesc_s_ch = idesc_bf16_f32(kBQ, kChunk, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kBQ, D, false, true);
      auto wait_slot = [&](uint32_t& addr) -> bool {
        if (!mbar_wait(&bars.kv_full[slot], phase, abort_flag, p.wait_ns)) return false;
        tc_fence_after();
        addr = smem_u32(sSlot + slot * C::SLOT);
        last = slot;
        if (++slot == (uint32_t)C::NSLOT) {
          slot = 0;
          phase ^= 1u;
        }
        return true;
      };
      auto release_slot = [&]() { mma_commit(&bars.kv_empty[last]); };
      // A descriptor's start-address field is the address in 16-byte units (the shared
      // window is below 256 KB, so the 14-bit field never carries): the descriptor of
      // a K-step is the tile's descriptor plus its byte offset / 16.
      const uint64_t qdesc0 = smem_desc_sw128(smem_u32(smem), 16, 1024);
      // S = Q K^T (K-major operands) into the stream's S buffer
      auto issue_s = [&](int x, uint32_t k_addr, int rows, uint32_t idesc) {
        const uint64_t a0 = qdesc0 + (uint64_t)((x * C::QBYTES) >> 4);
        const uint64_t b0 = smem_desc_sw128(k_addr, 16, 1024);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t adesc = a0 + (uint64_t)(((k / 4) * (kBQ * 128) + (k % 4) * 32) >> 4);
          const uint64_t bdesc = b0 + (uint64_t)(((k / 4) * (rows * 128) + (k % 4) * 32) >> 4);
          mma_ss(tmem + C::S_COL(x), adesc, bdesc, idesc, k > 0 ? 1u : 0u);
        }
      };
      // one step of stream x (see StreamPos); false when a wait gave up
      auto mstep = [&](StreamPos<C::QBPT, KP>& s, const int x) -> bool {
        if (s.t == 0) {
          // item start: its Q is loaded and the previous item's epilogue has read
          // this stream's S (first-order T) and O
          if (!mbar_wait(&bars.q_full[x], s.items & 1, abort_flag, p.wait_ns)) return false;
          if (s.items > 0 &&
              !mbar_wait(&bars.o_free[x], (s.items - 1) & 1, abort_flag, p.wait_ns))
            return false;
          tc_fence_after();
          if (s.n == 0) {
            mma_commit(&bars.o_final[x]);
            s.advance(p, x, n_ch);
            return true;
          }
          uint32_t k_addr;
          if (!wait_slot(k_addr)) return false;
          const bool chunk = 0 >= s.n_ex;
          issue_s(x, k_addr, chunk ? kChunk : C::KT, chunk ? idesc_s_ch : idesc_s_ex);
          release_slot();
          mma_commit(&bars.s_full[x]);
          s.t = 1;
          return true;
        }
        // PV(u) with P (bf16, TMEM) of tile u, then S(t): both operands' waits first, so
        // that the step's MMAs go out back to back
        const int u = s.t - 1;
        uint32_t v_addr, k_addr = 0;
        if (!wait_slot(v_addr)) return false;
        const uint32_t v_slot = last;
        const bool more = s.t < s.n;
        if (more && !wait_slot(k_addr)) return false;
        if (!mbar_wait(&bars.p_full[x], (s.tiles + u) & 1, abort_flag, p.wait_ns)) return false;
        tc_fence_after();
        {
          const int kdim = u >= s.n_ex ? kChunk : C::KT;
          const uint64_t b0 = smem_desc_sw128(v_addr, kdim * 128, 1024);
          // P of a kdim-key tile: half h (keys [h kdim/2, (h+1) kdim/2)) is packed at the
          // start of its own score columns, column h kdim/2 of the tile
          for (int k = 0; k < kdim / 16; ++k) {
            const int key = 16 * k, half = key / (kdim / 2);
            const uint32_t pcol = half * (kdim / 2) + (key - half * (kdim / 2)) / 2;
            mma_ts(tmem + C::O_COL(x), tmem + C::S_COL(x) + pcol, b0 + (uint64_t)(k * 128),
                   idesc_o, (u > 0 || k > 0) ? 1u : 0u);
          }
        }
        if (more) {
          const bool chunk = s.t >= s.n_ex;
          issue_s(x, k_addr, chunk ? kChunk : C::KT, chunk ? idesc_s_ch : idesc_s_ex);
          mma_commit(&bars.kv_empty[v_slot]);
          release_slot();
          mma_commit(&bars.s_full[x]);
          ++s.t;
          return true;
        }
        mma_commit(&bars.kv_empty[v_slot]);
        if (p.pisa) {
          // first-order term T = Q Hbar into this stream's (now free) S buffer
          uint32_t h_addr;
          if (!wait_slot(h_addr)) return false;
          const uint64_t a0 = qdesc0 + (uint64_t)((x * C::QBYTES) >> 4);
          const uint64_t b0 = smem_desc_sw128(h_addr, D * 128, 1024);
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            mma_ss(tmem + C::S_COL(x),
                   a0 + (uint64_t)(((k / 4) * (kBQ * 128) + (k % 4) * 32) >> 4),
                   b0 + (uint64_t)(k * 128), idesc_o, k > 0 ? 1u : 0u);
          release_slot();
        }
        mma_commit(&bars.o_final[x]);
        s.advance(p, x, n_ch);
        return true;
      };
      StreamPos<C::QBPT, KP> s0, s1;
      s0.k = s1.k = 0;
      s0.tiles = s1.tiles = 0;
      s0.items = s1.items = 0;
      s0.start(p, 0, n_ch);
      s1.start(p, 1, n_ch);
      while (ok && (s0.active(p) || s1.active(p))) {
        if (s0.active(p) && !(ok = mstep(s0, 0))) break;
        if (s1.active(p) && !(ok = mstep(s1, 1))) break;
      }
      // every issued MMA must complete before TMEM is released
      mma_commit(&bars.done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&bars.done, 0) && globaltimer_ns() - t0 < 100000000ull) {
      }
    }
    __syncwarp();
  } else {
    // ============================================ softmax + epilogue (per stream and half)
    const int x = warp / (4 * kHalves);        // stream
    const int hf = (warp / 4) % kHalves;       // column half
    const int quad = warp % 4;                 // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;          // query row within the tile
    const int bar_id = 1 + x;                  // the stream's named barrier (256 threads)
    constexpr int kPair = 128 * kHalves;
    const bool q_loader = hf == 0 && quad == 0 && lane == 0;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const uint32_t s_base = tmem + lane_addr + C::S_COL(x);
    const uint32_t o_half = tmem + lane_addr + C::O_COL(x) + hf * C::HALF_D;
    unsigned char* sq = smem + x * C::QBYTES;
    auto load_q = [&](int item) {
      int bh, qt;
      item_tile(p, item, bh, qt);
      mbar_arrive_expect_tx(&bars.q_full[x], p.qbox * D * 2);
      if (p.qbox == kBQ) {
        tma_load_4d(sq, &tmQ, &bars.q_full[x], 0, qt * kBQ, 0, bh);
      } else {  // L < 128: one box per column group, at the 128-row sub-tile stride
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tma_load_4d(sq + h * kBQ * 128, &tmQ, &bars.q_full[x], 0, 0, h, bh);
      }
    };
    int q_issued = 0;
    if (q_loader && stream_item(0, x) < p.n_items) {
      load_q(stream_item(0, x));
      q_issued = 1;
    }
    uint32_t tiles = 0;
    bool ok = true;
    for (int k = 0; stream_item(k, x) < p.n_items && ok; ++k) {
      const int item = stream_item(k, x);
      int bh, qt;
      item_tile(p, item, bh, qt);
      const Lists lists = item_lists<C::QBPT>(p.row_ptr, p.col_idx, p.csr_per_head, p.M, bh, qt);
      Steps<KP> steps;
      steps.init(lists);
      const int n_ex = count_steps<KP, C::QBPT>(lists);
      const int n = n_ex + n_ch;
      const int row_g = qt * kBQ + row;
      const int iq = qt * C::QBPT + row / BKV;   // this row's query block
      const bool has_blk = iq < p.M;
      const int32_t* rp = p.csr_per_head ? p.row_ptr + (size_t)bh * (p.M + 1) : p.row_ptr;
      const int mb = has_blk ? __ldg(rp + iq) : 0;
      const int me = has_blk ? __ldg(rp + iq + 1) : 0;
      int mp = mb;
      // this half's partial sums: l of the bf16 P (normalisation), le of the fp32 P
      // (log-sum-exp), sa of the bf16 centroid weights
      float m_run = -INFINITY, l = 0.f, le = 0.f, sa = 0.f;

      for (int t = 0; t < n; ++t) {
        const bool chunk = t >= n_ex;
        // this half's columns: [c0, c0 + w) of the tile
        const int w = chunk ? 64 : C::HALF_EX;
        const int c0 = hf * w;
        uint32_t ex0 = 0u, ex1 = 0u;   // excluded columns of the half
        bool masked = false, skip = false;
        if (chunk) {
          // centroid chunk: exclude this row's selected blocks and the indices past M.
          // The 32 rows of a warp share one query block, so the lanes read its list
          // together (coalesced) and OR their bits across the warp; this runs before the
          // wait for S, which hides the loads' latency
          const int base = (t - n_ex) * kChunk + c0;
          uint32_t w0 = 0u, w1 = 0u;
          for (int e0 = mb; e0 < me; e0 += 32) {
            const int e = e0 + lane;
            const int cj = e < me ? __ldg(p.col_idx + e) - base : -1;
            if (cj >= 0 && cj < 64) {
              const uint32_t bit = 1u << (cj & 31);
              w0 |= cj < 32 ? bit : 0u;
              w1 |= cj >= 32 ? bit : 0u;
            }
          }
          uint32_t t0, t1;
          tail_bits(has_blk ? p.M - base : 0, t0, t1);
          ex0 = __reduce_or_sync(kAll, w0) | t0;
          ex1 = __reduce_or_sync(kAll, w1) | t1;
          masked = true;
        } else {
          int jt = -1;   // key block of this half (needed for membership and padding)
          if (C::QBPT == 2 && KP) {
            // a pair of blocks: this row's own list may hold either; the half of the
            // block it lacks is skipped
            const int b0 = 2 * steps.next();
            const bool in0 = mp < me && __ldg(p.col_idx + mp) == b0;
            if (in0) ++mp;
            const bool in1 = mp < me && __ldg(p.col_idx + mp) == b0 + 1;
            if (in1) ++mp;
            jt = b0 + hf;
            skip = !(hf ? in1 : in0);
          } else if (C::QBPT == 2) {
            jt = steps.next();
            const bool member = mp < me && __ldg(p.col_idx + mp) == jt;
            if (member) ++mp;
            skip = !member;
          } else if (p.key_valid != nullptr) {
            jt = __ldg(p.col_idx + mb + t);   // one query block per tile: its own list
          }
          // token padding: an exact tile of a block with fewer real tokens than its width
          // excludes its tail columns
          if (!skip && p.key_valid != nullptr && jt >= 0) {
            // (with KP the half is the whole block)
            const int v = min(max(__ldg(p.key_valid + jt), 1), BKV) - (KP ? 0 : c0);
            if (v < w) {
              masked = true;
              tail_bits(v, ex0, ex1);
            }
          }
        }
        const bool got = mbar_wait(&bars.s_full[x], (tiles + t) & 1, abort_flag, p.wait_ns);
        // pass 1: this half's row max over its w columns, 32 at a time. With w = 64 the
        // upper chunk is read first and the lower one kept in registers for pass 2.
        const uint32_t a = s_base + c0;
        uint32_t r[32];
        float mh = -INFINITY;
        if (got && !skip) {
          tc_fence_after();
          if (w == 64) {
            tmem_ld32(a + 32, r);
            tmem_wait_ld();
            if (masked) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if ((ex1 >> e) & 1u) r[e] = __float_as_uint(-INFINITY);
            }
            mh = row_max<32, 32>(r);
          }
          tmem_ld32(a, r);
          tmem_wait_ld();
          if (masked) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if ((ex0 >> e) & 1u) r[e] = __float_as_uint(-INFINITY);
          }
          mh = fmaxf(mh, row_max<32, 32>(r));
        }
        // the pair's max: both halves' maxima (as bf16) through shared memory. The
        // barrier also agrees on leaving when a wait gave up. The next tile's write comes
        // after the next S, which the MMA issuer starts only after both halves' P.
        const uint16_t mine = bf16_bits(mh * p.scale_log2);
        s_max[x][hf][row] = mine;
        ok = bar_and(bar_id, kPair, got);
        if (!ok) break;
        const float mx = fmaxf(bf16_value(mine), bf16_value(s_max[x][hf ^ 1][row]));
        const bool need = mx > m_run + kRescaleLog2;
        if (__any_sync(kAll, need)) {
          const float m_new = need ? mx : m_run;
          const float factor = need ? ex2(m_run - m_new) : 1.0f;
          if (t > 0) {
            // PV(t-1) was issued before S(t), so it has completed: rescale this half of O
#pragma unroll 1
            for (int c = 0; c < C::HALF_D; c += 16) {
              uint32_t ro[16];
              tmem_ld16(o_half + c, ro);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) ro[e] = __float_as_uint(__uint_as_float(ro[e]) * factor);
              tmem_st16(o_half + c, ro);
            }
            tmem_wait_st();
          }
          l *= factor;
          le *= factor;
          sa *= factor;
          m_run = m_new;
        }
        const float m_ref = m_run == -INFINITY ? 0.f : m_run;
        // pass 2: P = 2^(s*scale_log2 - m) as bf16 pairs, packed at the start of this
        // half's own columns (16 columns per 32 scores). The lower chunk, in registers,
        // goes over its own first 16 columns; then the upper chunk is read again (no P
        // has been written over it) and goes over the lower chunk's last 16 columns.
        float2 rs = make_float2(0.f, 0.f);
        if (skip) {
          uint32_t z[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) z[e] = 0u;
          for (int c = 0; c < w / 2; c += 8) tmem_st8(a + c, z);
        } else {
          rs = masked ? half_exp<32, true, true>(r, p.scale_log2, m_ref, a)
                      : half_exp<32, true, false>(r, p.scale_log2, m_ref, a);
          if (w == 64) {
            tmem_ld32(a + 32, r);
            tmem_wait_ld();
            if (masked) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if ((ex1 >> e) & 1u) r[e] = __float_as_uint(-INFINITY);
            }
            const float2 r2 = masked ? half_exp<32, true, true>(r, p.scale_log2, m_ref, a + 16)
                                     : half_exp<32, true, false>(r, p.scale_log2, m_ref, a + 16);
            rs = make_float2(rs.x + r2.x, rs.y + r2.y);
          }
        }
        if (chunk) {
          l += (float)BKV * rs.x;
          le += (float)BKV * rs.y;
          sa += rs.x;
        } else {
          l += rs.x;
          le += rs.y;
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars.p_full[x]);
      }
      if (!ok) break;

      // ---------------------------------------------------------------- epilogue
      const bool fin = mbar_wait(&bars.o_final[x], k & 1, abort_flag, p.wait_ns);
      // every MMA of this item has completed: the Q buffer is free. The pair first adds
      // its partial sums through it (half 0's first, in both halves, so that they agree
      // to the bit), then stages this tile's output there for one TMA store.
      float* xsum = reinterpret_cast<float*>(sq);   // [half][row][4]
      xsum[(hf * kBQ + row) * 4] = l;
      xsum[(hf * kBQ + row) * 4 + 1] = sa;
      xsum[(hf * kBQ + row) * 4 + 2] = le;
      ok = bar_and(bar_id, kPair, fin);
      if (!ok) break;
      tc_fence_after();
      const float l_o = xsum[((hf ^ 1) * kBQ + row) * 4];
      const float sa_o = xsum[((hf ^ 1) * kBQ + row) * 4 + 1];
      const float le_o = xsum[((hf ^ 1) * kBQ + row) * 4 + 2];
      const float l_all = hf == 0 ? l + l_o : l_o + l;
      const float sa_all = hf == 0 ? sa + sa_o : sa_o + sa;
      const float le_all = hf == 0 ? le + le_o : le_o + le;
      bar_sync(bar_id, kPair);   // both halves have read the sums: the buffer is free
      const bool tma_out = p.qbox == kBQ;
      if (!tma_out && q_loader && stream_item(k + 1, x) < p.n_items) {
        load_q(stream_item(k + 1, x));
        ++q_issued;
      }
      const bool write = row_g < p.L;
      __nv_bfloat16* orow = p.O + ((size_t)bh * p.L + (write ? row_g : 0)) * D;
      const float inv_l = l_all > 0.f ? 1.0f / l_all : 0.f;
      const float c1 = p.scale * sa_all;
#pragma unroll 1
      for (int cc = 0; cc < C::HALF_D; cc += 8) {
        const int c = hf * C::HALF_D + cc;   // column of O
        uint32_t ro[8], rt[8];
        if (n > 0) {
          tmem_ld8(o_half + cc, ro);
          if (p.pisa) tmem_ld8(s_base + c, rt);  // T = Q Hbar sits in the S buffer
          tmem_wait_ld();
        }
        uint32_t packed[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          float a0 = 0.f, a1 = 0.f;
          if (n > 0) {
            a0 = __uint_as_float(ro[e]);
            a1 = __uint_as_float(ro[e + 1]);
            if (p.pisa) {
              a0 = fmaf(c1, __uint_as_float(rt[e]), a0);
              a1 = fmaf(c1, __uint_as_float(rt[e + 1]), a1);
            }
          }
          packed[e / 2] = pack_bf16x2(a0 * inv_l, a1 * inv_l);
        }
        const uint4 v4 = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        if (tma_out) {
          // 128-byte swizzle of the Q layout: 16-byte chunk j of row r sits at j ^ (r % 8)
          const int j = (c % 64) / 8;
          *reinterpret_cast<uint4*>(sq + (c / 64) * (kBQ * 128) + row * 128 +
                                    ((j ^ (row & 7)) * 16)) = v4;
        } else if (write) {
          *reinterpret_cast<uint4*>(orow + c) = v4;
        }
      }
      bool staged = true;
      if (tma_out) {
        fence_proxy_async_smem();
        mbar_arrive(&bars.o_staged[x]);  // this half row is staged
        if (q_loader) {
          staged = mbar_wait(&bars.o_staged[x], k & 1, abort_flag, p.wait_ns);
          if (staged) {
            tma_store_4d(&tmO, sq, 0, qt * kBQ, 0, bh);  // rows past L are not written
            bulk_commit_group();
            bulk_wait_read_all();
            if (stream_item(k + 1, x) < p.n_items) {
              load_q(stream_item(k + 1, x));
              ++q_issued;
            }
          }
        }
      }
      if (hf == 0 && write && p.lse)
        p.lse[(size_t)bh * p.L + row_g] =
            le_all > 0.f ? (m_run + log2f(le_all)) * 0.69314718055994531f : -INFINITY;
      tc_fence_before();
      mbar_arrive(&bars.o_free[x]);
      tiles += n;
      ok = bar_and(bar_id, kPair, staged);
    }
    if (q_loader) bulk_wait_all();  // this stream's output stores have completed
    if (!ok && q_loader && q_issued > 0) {
      // drain this stream's last Q copy (bounded) before the CTA exits
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&bars.q_full[x], (q_issued - 1) & 1) &&
             globaltimer_ns() - t0 < 100000000ull) {
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && abort_sh) report(p.status, BSA_ERR_TIMEOUT);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int BKV, bool KP>
cudaError_t run(const ForwardArgs& a, const int32_t* flag, const void* kb16, const void* vs16,
                const void* hb16, int Mp, cudaStream_t st) {
  using C = Cfg<D, BKV, KP>;
  const Shape& s = a.s;
  const int BH = s.BH(), M = s.M();
  CUtensorMap tmQ, tmK, tmV, tmKb, tmVs, tmHb, tmO;
  const int qbox = s.L < kBQ ? s.L : kBQ;
  bool ok = make_map(&tmQ, a.Q, D, s.L, BH, qbox, qbox == kBQ) &&
            make_map(&tmK, a.K, D, s.L, BH, C::KT) && make_map(&tmV, a.V, D, s.L, BH, C::KT);
  // the output map (128-row boxes) is used only when every query tile is 128 rows
  if (qbox == kBQ) ok = ok && make_map(&tmO, a.O, D, s.L, BH, kBQ);
  else tmO = tmQ;
  const bool pisa = a.mode == BSA_MODE_PISA;
  if (pisa) {
    ok = ok && make_map(&tmKb, kb16, D, Mp, BH, kChunk) &&
         make_map(&tmVs, vs16, D, Mp, BH, kChunk) && make_map(&tmHb, hb16, D, D, BH, D);
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
  p.tile_major = a.csr_per_head ? 0 : 1;
  p.qbox = qbox;
  p.row_ptr = a.row_ptr;
  p.col_idx = a.col_idx;
  p.csr_per_head = a.csr_per_head;
  p.pisa = pisa;
  p.key_valid = s.key_valid;
  p.scale = a.scale;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.O = static_cast<__nv_bfloat16*>(a.O);
  p.lse = a.lse;
  p.flag = flag;
  p.status = a.status;
  p.wait_ns = a.wait_ns > 0 ? a.wait_ns : kWaitTimeoutNs;
  cudaError_t e = cudaFuncSetAttribute(k_pair<D, BKV, KP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int grid = min(p.n_items, sm_count());
  k_pair<D, BKV, KP><<<grid, kThreads, C::SMEM, st>>>(tmQ, tmK, tmV, tmKb, tmVs, tmHb, tmO, p);
  return cudaGetLastError();
}

}  // namespace fwdpair

cudaError_t launch_forward_pair(const ForwardArgs& a, const int32_t* flag, const void* kb16,
                                const void* vs16, const void* hb16, int Mp, cudaStream_t st) {
  // instantiated for head dim 64 only, the shape it is dispatched for
  const Shape& s = a.s;
  if (s.d != 64) return cudaErrorInvalidValue;
  // 64-token blocks go two to a 128-key step once the sequence holds a whole step (a
  // K/V box of 128 rows must fit in the tensor)
  if (s.block == 64 && s.L >= fwdpair::kBQ) return fwdpair::run<64, 64, true>(a, flag, kb16, vs16, hb16, Mp, st);
  if (s.block == 64) return fwdpair::run<64, 64, false>(a, flag, kb16, vs16, hb16, Mp, st);
  return fwdpair::run<64, 128, false>(a, flag, kb16, vs16, hb16, Mp, st);
}

}  // namespace bsa
