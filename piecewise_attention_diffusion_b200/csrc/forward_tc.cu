// bsa_forward on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), sm_100a: the
// kernel for head dim 128 in the keep-or-drop and PISA modes, and for every head dim in
// the per-block first-order mode (head dim 64 in the other two modes runs the kernel of
// forward_pair.cu). This file also holds the launch dispatch and the statistics
// conversion to bf16.
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
// Design (one persistent CTA per SM, 384 threads, warp-specialised, two query tiles in
// flight so that the softmax of one overlaps the tensor-core work of the other):
//   warps 0-3, 4-7  one softmax warpgroup per stream: thread r owns query row r (TMEM
//           lane r). The whole S row is loaded into registers with one wait; the row max
//           uses three-input max; P = 2^(s*scale*log2(e) - m) is formed with packed f32x2
//           arithmetic, a quarter of the exponentials on the FMA pipe (polynomial) and the
//           rest on the special-function unit, so that neither pipe limits alone; P goes
//           back into TMEM as bf16 pairs with tcgen05.st. O is rescaled in TMEM only when
//           the running max grows by more than 2^8 (keeps every P <= 256, safe in bf16 and
//           fp32). The same warps run the epilogue and load the next query tile of their
//           stream;
//   warp 8  TMA producer of a ring of K / V / centroid / Hbar tiles (128-byte swizzled,
//           completion on mbarriers), in the same step order as the MMA issuer;
//   warp 9  MMA issuer (one thread), alternating one step of each stream:
//           step 0 = S(0); step t = O += P(t-1) V(t-1), then S(t) = Q K(t)^T; last step =
//           O += P(n-1) V(n-1) [, T = Q Hbar]. P is bf16 in TMEM over its own S buffer and
//           is the A operand of the PV product. Because S(t) is issued after PV(t-1) in
//           the same stream, S(t) being ready implies PV(t-1) has completed;
//   warps 10-11  idle (they complete the control warpgroup, whose registers setmaxnreg
//           hands to the softmax warpgroups).
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256, 256+D), O1 [256+D, 256+2D); the
// first-order product T of a stream is written into its S buffer after its last PV.
// Query tiles are 128 rows: one query block of 128, or two of 64 whose key-block lists
// are merged (each row masks the key blocks its own block does not select).
// Every mbarrier wait is bounded (sm100::mbar_wait); on a timeout the CTA drains its
// in-flight copies and MMAs, frees TMEM and reports BSA_ERR_TIMEOUT.
#include <limits.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "forward_tiles.cuh"
#include "sm100.cuh"

namespace bsa {
namespace fwdtc {

using namespace sm100;
using namespace fwdtiles;

constexpr int kBQ = 128;       // query rows per tile
constexpr int kChunk = 128;    // centroids per sweep tile
constexpr int kStreams = 2;                   // query tiles in flight per CTA
static_assert(kStreams == 2, "the issuer's Q descriptor table holds two streams");
constexpr int kThreads = 128 * (kStreams + 1);  // softmax warpgroups, then a control warpgroup
constexpr int kProducerWarp = 4 * kStreams;      // first warp of the control warpgroup
constexpr int kMmaWarp = kProducerWarp + 1;      // (its two other warps only idle)
// Register split: the launch gives every thread 168 registers (3 warps per SMSP); the
// control warpgroup drops to 88 and the softmax warpgroups rise to 208, which hold a whole
// S row: 128 x 88 + 256 x 208 = 384 x 168.
constexpr int kRegsControl = 88;
constexpr int kRegsSoftmax = 208;
static_assert(128 * kRegsControl + 128 * kStreams * kRegsSoftmax <= kThreads * 168, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

struct Params {
  int L, M, BH, n_qt, n_items;
  int tile_major;  // items ordered (tile, head) instead of (head, tile): lists shared by all heads
  int qbox;  // rows per Q box: 128, or L when L < 128
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int csr_per_head;
  int pisa;
  int linear;  // per-block first order: every block a tile, unselected ones linearised
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

template <int D, int BKV>
struct Cfg {
  static constexpr int QBPT = kBQ / BKV;          // query blocks per tile (1 or 2)
  static constexpr int QBYTES = kBQ * D * 2;
  static constexpr int SLOT = kBQ * D * 2;        // a slot holds up to 128 rows x D
  static constexpr int NSLOT = D == 128 ? 5 : 8;
  static constexpr int SMEM = kStreams * QBYTES + NSLOT * SLOT + 1024;
  // TMEM columns: S of stream x at 128x, O of stream x at 256 + D*x
  __host__ __device__ static constexpr uint32_t S_COL(int x) { return 128u * x; }
  __host__ __device__ static constexpr uint32_t O_COL(int x) { return 256u + D * x; }
};

// Work item k of stream x of this CTA (static schedule: the CTA takes items
// blockIdx.x, blockIdx.x + G, ... and deals them to its two streams alternately).
__device__ __forceinline__ int stream_item(int k, int x) {
  return blockIdx.x + (2 * k + x) * gridDim.x;
}

// Per-stream position in the step schedule shared by the producer and the MMA issuer.
// Steps of an item with n tiles: step 0 = S(0); step t (1 <= t < n) = PV(t-1), S(t);
// step n = PV(n-1) [+ T] and the end of the item. An item with n = 0 has one step.
template <int QBPT>
struct StreamPos {
  int k, item, bh, qt, n, n_ex, t;
  uint32_t tiles;  // tiles of earlier items of this stream (barrier phases)
  int items;       // earlier items of this stream
  Lists lk, lv;    // K-side and V-side list cursors (producer)
  __device__ __forceinline__ void start(const Params& p, int x, int n_ch) {
    item = stream_item(k, x);
    if (item >= p.n_items) return;
    item_tile(p, item, bh, qt);
    lk = item_lists<QBPT>(p.row_ptr, p.col_idx, p.csr_per_head, p.M, bh, qt);
    lv = lk;
    n_ex = p.linear ? p.M : count_exact<QBPT>(lk);
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

struct Barriers {
  uint64_t kv_full[8], kv_empty[8];
  uint64_t q_full[kStreams];
  uint64_t s_full[kStreams], p_full[kStreams];
  uint64_t o_final[kStreams], o_free[kStreams], o_staged[kStreams];
  uint64_t done;
};

template <int D, int BKV, bool kLinear>
__global__ void __launch_bounds__(kThreads, 1)
k_forward(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
          const __grid_constant__ CUtensorMap tmVs, const __grid_constant__ CUtensorMap tmHb,
          const __grid_constant__ CUtensorMap tmO, const Params p) {
  using C = Cfg<D, BKV>;
  if (*p.flag) return;  // malformed lists: leave O untouched

  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sSlot = smem + kStreams * C::QBYTES;
  __shared__ Barriers bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int x = 0; x < kStreams; ++x) {
      mbar_init(&bars.q_full[x], 1);
      mbar_init(&bars.s_full[x], 1);
      mbar_init(&bars.p_full[x], 128);
      mbar_init(&bars.o_final[x], 1);
      mbar_init(&bars.o_free[x], 128);
      mbar_init(&bars.o_staged[x], 128);
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
  if (warp >= kProducerWarp) {
  setmaxnreg_dec<kRegsControl>();
  if (warp == kProducerWarp) {
    // ================================================= TMA producer of the K/V ring
    if (lane == 0) {
      uint32_t ring = 0;
      bool ok = true;
      auto tile_map = [&](int kind, int j, const CUtensorMap*& map, int& y, int& rows) {
        map = kind == kLoadK ? &tmK : kind == kLoadV ? &tmV : kind == kLoadKbar ? &tmKb
              : kind == kLoadVsum ? &tmVs : &tmHb;
        rows = kind <= kLoadV ? BKV : (kind == kLoadHbar ? D : kChunk);
        y = kind <= kLoadV ? j * BKV : (kind == kLoadHbar ? 0 : j * kChunk);
      };
      auto load = [&](int kind, int j, int bh) -> bool {
        const int slot = ring % C::NSLOT;
        const uint32_t ph = (ring / C::NSLOT) & 1;
        if (!mbar_wait(&bars.kv_empty[slot], ph ^ 1, abort_flag, p.wait_ns)) return false;
        unsigned char* dst = sSlot + slot * C::SLOT;
        const CUtensorMap* map;
        int y, rows;
        tile_map(kind, j, map, y, rows);
        mbar_arrive_expect_tx(&bars.kv_full[slot], rows * D * 2);
        // one 4-D box: 64 columns x rows x (D/64) column groups; lands as D/64 swizzled
        // [rows x 64] sub-tiles, sub-tile h at byte offset h * rows * 128
        tma_load_4d(dst, map, &bars.kv_full[slot], 0, y, 0, bh);
        ++ring;
        return true;
      };
      // the loads of one step of stream x, in the MMA issuer's order
      auto step = [&](StreamPos<C::QBPT>& s, int x) -> bool {
        if (s.t == 0) {
          if (s.n == 0) {
            s.advance(p, x, n_ch);
            return true;
          }
          const bool r = s.n_ex > 0 ? load(kLoadK, p.linear ? 0 : s.lk.next(), s.bh)
                                    : load(kLoadKbar, 0, s.bh);
          s.t = 1;
          return r;
        }
        const int u = s.t - 1;
        if (!(u < s.n_ex ? load(kLoadV, p.linear ? u : s.lv.next(), s.bh)
                         : load(kLoadVsum, u - s.n_ex, s.bh)))
          return false;
        if (s.t < s.n) {
          const bool r = s.t < s.n_ex ? load(kLoadK, p.linear ? s.t : s.lk.next(), s.bh)
                                      : load(kLoadKbar, s.t - s.n_ex, s.bh);
          ++s.t;
          return r;
        }
        const bool r = p.pisa ? load(kLoadHbar, 0, s.bh) : true;
        s.advance(p, x, n_ch);
        return r;
      };
      StreamPos<C::QBPT> s0, s1;
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
      constexpr uint32_t idesc_s_ex = idesc_bf16_f32(kBQ, BKV, false, false);
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
      const uint64_t qdesc[kStreams] = {smem_desc_sw128(smem_u32(smem), 16, 1024),
                                        smem_desc_sw128(smem_u32(smem + C::QBYTES), 16, 1024)};
      // S = Q K^T (K-major operands) into the stream's S buffer
      auto issue_s = [&](int x, uint32_t k_addr, int rows, uint32_t idesc) {
        const uint64_t a0 = x ? qdesc[1] : qdesc[0];
        const uint64_t b0 = smem_desc_sw128(k_addr, 16, 1024);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t adesc = a0 + (uint64_t)(((k / 4) * (kBQ * 128) + (k % 4) * 32) >> 4);
          const uint64_t bdesc = b0 + (uint64_t)(((k / 4) * (rows * 128) + (k % 4) * 32) >> 4);
          mma_ss(tmem + C::S_COL(x), adesc, bdesc, idesc, k > 0 ? 1u : 0u);
        }
      };
      // one step of stream x (see StreamPos); false when a wait gave up
      auto mstep = [&](StreamPos<C::QBPT>& s, const int x) -> bool {
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
          issue_s(x, k_addr, chunk ? kChunk : BKV, chunk ? idesc_s_ch : idesc_s_ex);
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
          const int kdim = u >= s.n_ex ? kChunk : BKV;
          const uint64_t b0 = smem_desc_sw128(v_addr, kdim * 128, 1024);
          for (int k = 0; k < kdim / 16; ++k)
            mma_ts(tmem + C::O_COL(x), tmem + C::S_COL(x) + k * 8, b0 + (uint64_t)(k * 128),
                   idesc_o, (u > 0 || k > 0) ? 1u : 0u);
        }
        if (more) {
          const bool chunk = s.t >= s.n_ex;
          issue_s(x, k_addr, chunk ? kChunk : BKV, chunk ? idesc_s_ch : idesc_s_ex);
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
          const uint64_t a0 = x ? qdesc[1] : qdesc[0];
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
      StreamPos<C::QBPT> s0, s1;
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
  }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // ==================================================== softmax + epilogue (per stream)
    const int x = warp / 4;                    // stream of this warpgroup
    const int quad = warp % 4;                 // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;          // query row within the tile
    const bool q_loader = quad == 0 && lane == 0;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const uint32_t s_base = tmem + lane_addr + C::S_COL(x);
    const uint32_t o_base = tmem + lane_addr + C::O_COL(x);
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
      Lists lists = item_lists<C::QBPT>(p.row_ptr, p.col_idx, p.csr_per_head, p.M, bh, qt);
      const int n_ex = kLinear ? p.M : count_exact<C::QBPT>(lists);
      const int n = n_ex + n_ch;
      const int row_g = qt * kBQ + row;
      const int iq = qt * C::QBPT + row / BKV;   // this row's query block
      const bool has_blk = iq < p.M;
      const int32_t* rp = p.csr_per_head ? p.row_ptr + (size_t)bh * (p.M + 1) : p.row_ptr;
      const int mb = has_blk ? __ldg(rp + iq) : 0;
      const int me = has_blk ? __ldg(rp + iq + 1) : 0;
      int mp = mb;
      // per-block first order: the row's next selected block, fetched one match ahead
      int nxt = kLinear && mp < me ? __ldg(p.col_idx + mp) : INT_MAX;
      float m_run = -INFINITY, l = 0.f, sa = 0.f;

      for (int t = 0; t < n; ++t) {
        const bool chunk = t >= n_ex;
        uint32_t excl[4] = {0u, 0u, 0u, 0u};
        if (chunk) {
          // centroid chunk: exclude this row's selected blocks and the indices past M.
          // The 32 rows of a warp share one query block, so the lanes read its list
          // together (coalesced) and OR their bits across the warp; this runs before the
          // wait for S, which hides the loads' latency
          const int base = (t - n_ex) * kChunk;
          uint32_t w0 = 0u, w1 = 0u, w2 = 0u, w3 = 0u;
          for (int e0 = mb; e0 < me; e0 += 32) {
            const int e = e0 + lane;
            const int cj = e < me ? __ldg(p.col_idx + e) - base : -1;
            if (cj >= 0 && cj < kChunk) {
              const uint32_t bit = 1u << (cj & 31);
              const int wd = cj >> 5;
              w0 |= wd == 0 ? bit : 0u;
              w1 |= wd == 1 ? bit : 0u;
              w2 |= wd == 2 ? bit : 0u;
              w3 |= wd == 3 ? bit : 0u;
            }
          }
          excl[0] = __reduce_or_sync(0xffffffffu, w0);
          excl[1] = __reduce_or_sync(0xffffffffu, w1);
          excl[2] = __reduce_or_sync(0xffffffffu, w2);
          excl[3] = __reduce_or_sync(0xffffffffu, w3);
          const int valid = has_blk ? min(kChunk, p.M - base) : 0;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int lo = w * 32;
            if (valid <= lo) excl[w] = 0xffffffffu;
            else if (valid < lo + 32) excl[w] |= 0xffffffffu << (valid - lo);
          }
        }
        bool skip = false;          // whole tile masked for this row
        bool lin = false;           // block t unselected for this row (per-block mode)
        int jt = -1;                // key block of an exact tile (needed with padding)
        if (kLinear) {
          jt = t;
          if (nxt == t) {
            ++mp;
            nxt = mp < me ? __ldg(p.col_idx + mp) : INT_MAX;
          } else {
            lin = true;
          }
        } else if (!chunk && C::QBPT == 2) {
          jt = lists.next();
          const bool member = mp < me && __ldg(p.col_idx + mp) == jt;
          if (member) ++mp;
          skip = !member;
        } else if (!chunk && p.key_valid != nullptr) {
          jt = __ldg(p.col_idx + mb + t);   // one query block per tile: its own list
        }
        // token padding: an exact tile of a block with fewer real tokens than its width
        // excludes its tail columns (the same exclusion bits as a centroid chunk)
        bool masked = false;
        if (!chunk && p.key_valid != nullptr && jt >= 0) {
          const int v = min(max(__ldg(p.key_valid + jt), 1), BKV);
          if (v < BKV) {
            masked = true;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const int lo = w * 32;
              excl[w] = v <= lo ? 0xffffffffu : (v < lo + 32 ? 0xffffffffu << (v - lo) : 0u);
            }
          }
        }
        ok = mbar_wait(&bars.s_full[x], (tiles + t) & 1, abort_flag, p.wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        // pass 1: this thread's whole S row into registers (one wait), the excluded
        // entries of a centroid chunk set to -inf, then the row max
        const int cols = chunk ? kChunk : BKV;
        uint32_t r[128];
        float mx = -INFINITY;
        if (!skip) {
          tmem_ld32(s_base, *reinterpret_cast<uint32_t(*)[32]>(r));
          tmem_ld32(s_base + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
          if (cols == 128) {
            tmem_ld32(s_base + 64, *reinterpret_cast<uint32_t(*)[32]>(r + 64));
            tmem_ld32(s_base + 96, *reinterpret_cast<uint32_t(*)[32]>(r + 96));
          }
          tmem_wait_ld();
          if (chunk || masked) {
#pragma unroll
            for (int e = 0; e < 128; ++e)
              if ((excl[e >> 5] >> (e & 31)) & 1u) r[e] = __float_as_uint(-INFINITY);
          }
          if (kLinear && lin)  // the block's centroid score: the mean of its row scores
            mx = (BKV == 128 ? row_sum<128, 128>(r) : row_sum<64, 128>(r)) * (1.0f / BKV);
          else
            mx = cols == 128 ? row_max<128, 128>(r) : row_max<64, 128>(r);
        }
        const float mean = mx;
        mx *= p.scale_log2;
        const bool need = mx > m_run + kRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          const float m_new = need ? mx : m_run;
          const float factor = need ? ex2(m_run - m_new) : 1.0f;
          if (t > 0) {
            // PV(t-1) was issued before S(t), so it has completed: rescale O in TMEM
#pragma unroll 1
            for (int c = 0; c < D; c += 16) {
              uint32_t ro[16];
              tmem_ld16(o_base + c, ro);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) ro[e] = __float_as_uint(__uint_as_float(ro[e]) * factor);
              tmem_st16(o_base + c, ro);
            }
            tmem_wait_st();
          }
          l *= factor;
          sa *= factor;
          m_run = m_new;
        }
        const float m_ref = m_run == -INFINITY ? 0.f : m_run;
        // pass 2: P = 2^(s*scale_log2 - m) as bf16 pairs over the first cols/2 columns of
        // the S buffer (the row is in registers, so the overwrite is safe)
        float rs = 0.f;
        if (skip) {
          uint32_t z[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) z[e] = 0u;
          tmem_st32(s_base, z);
          if (cols == 128) tmem_st32(s_base + 32, z);
        } else if (kLinear && lin) {
          // first-order weights about the centroid: alpha (1 + s (score - mean)); the
          // block adds B alpha to the denominator (its first-order part sums to zero)
          const float alpha = ex2(mx - m_ref);
          row_lin<BKV, 128>(r, alpha * p.scale, alpha * (1.0f - p.scale * mean), s_base);
          rs = (float)BKV * alpha;
        } else if (chunk) {
          rs = row_exp<128, false, 128>(r, p.scale_log2, m_ref, s_base);
        } else if (masked) {  // -inf entries: the special-function unit gives exact zeros
          rs = row_exp<BKV, false, 128>(r, p.scale_log2, m_ref, s_base);
        } else {
          rs = row_exp<BKV, true, 128>(r, p.scale_log2, m_ref, s_base);
        }
        if (chunk) {
          l += (float)BKV * rs;
          sa += rs;
        } else {
          l += rs;
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars.p_full[x]);
      }
      if (!ok) break;

      // ---------------------------------------------------------------- epilogue
      ok = mbar_wait(&bars.o_final[x], k & 1, abort_flag, p.wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // every MMA of this item has completed: Q's buffer is free. With full 128-row tiles
      // it first stages this tile's output for one TMA store (coalesced, asynchronous) and
      // takes the next Q after the store has read it; otherwise the next Q is loaded now
      // and every row is stored directly.
      const bool tma_out = p.qbox == kBQ;
      if (!tma_out && q_loader && stream_item(k + 1, x) < p.n_items) {
        load_q(stream_item(k + 1, x));
        ++q_issued;
      }
      const bool write = row_g < p.L;
      __nv_bfloat16* orow = p.O + ((size_t)bh * p.L + (write ? row_g : 0)) * D;
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      const float c1 = p.scale * sa;
#pragma unroll 1
      for (int c = 0; c < D; c += 16) {
        uint32_t ro[16], rt[16];
        if (n > 0) {
          tmem_ld16(o_base + c, ro);
          if (p.pisa) tmem_ld16(s_base + c, rt);  // T = Q Hbar sits in the S buffer
          tmem_wait_ld();
        }
        uint32_t packed[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
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
        if (tma_out) {
          // 128-byte swizzle of the Q layout: 16-byte chunk j of row r sits at j ^ (r % 8)
          const int j = (c % 64) / 8;
          unsigned char* rp_s = sq + (c / 64) * (kBQ * 128) + row * 128;
          *reinterpret_cast<uint4*>(rp_s + ((j ^ (row & 7)) * 16)) =
              make_uint4(packed[0], packed[1], packed[2], packed[3]);
          *reinterpret_cast<uint4*>(rp_s + (((j + 1) ^ (row & 7)) * 16)) =
              make_uint4(packed[4], packed[5], packed[6], packed[7]);
        } else if (write) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c);
          dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        }
      }
      if (tma_out) {
        fence_proxy_async_smem();
        mbar_arrive(&bars.o_staged[x]);  // this row is staged
        bool staged = true;
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
        ok = __all_sync(0xffffffffu, staged);
        if (!ok) break;
      }
      if (write && p.lse)
        p.lse[(size_t)bh * p.L + row_g] =
            l > 0.f ? (m_run + log2f(l)) * 0.69314718055994531f : -INFINITY;
      tc_fence_before();
      mbar_arrive(&bars.o_free[x]);
      tiles += n;
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
template <int D, int BKV, bool kLinear>
cudaError_t run(const ForwardArgs& a, const int32_t* flag, const void* kb16, const void* vs16,
                const void* hb16, cudaStream_t st) {
  using C = Cfg<D, BKV>;
  const Shape& s = a.s;
  const int BH = s.BH(), M = s.M();
  CUtensorMap tmQ, tmK, tmV, tmKb, tmVs, tmHb, tmO;
  const int qbox = s.L < kBQ ? s.L : kBQ;
  const int Mp = ceil_div(M, kChunk) * kChunk;
  bool ok = make_map(&tmQ, a.Q, D, s.L, BH, qbox, qbox == kBQ) &&
            make_map(&tmK, a.K, D, s.L, BH, BKV) &&
            make_map(&tmV, a.V, D, s.L, BH, BKV);
  // the output map (128-row boxes) is used only when every query tile is 128 rows
  if (qbox == kBQ) ok = ok && make_map(&tmO, a.O, D, s.L, BH, kBQ);
  else tmO = tmQ;
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
  p.tile_major = a.csr_per_head ? 0 : 1;
  p.qbox = qbox;
  p.row_ptr = a.row_ptr;
  p.col_idx = a.col_idx;
  p.csr_per_head = a.csr_per_head;
  p.pisa = a.mode == BSA_MODE_PISA;
  p.linear = a.mode == BSA_MODE_PISA_BLOCK;
  p.key_valid = s.key_valid;
  p.scale = a.scale;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.O = static_cast<__nv_bfloat16*>(a.O);
  p.lse = a.lse;
  p.flag = flag;
  p.status = a.status;
  p.wait_ns = a.wait_ns > 0 ? a.wait_ns : kWaitTimeoutNs;
  cudaError_t e = cudaFuncSetAttribute(k_forward<D, BKV, kLinear>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  // setmaxnreg.inc waits until the warpgroups that shrink have released enough registers:
  // the split must fit in what the launch allocates, or the kernel would never start
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, k_forward<D, BKV, kLinear>);
  if (e != cudaSuccess) return e;
  if (fa.numRegs * kThreads < 128 * kRegsControl + 128 * kStreams * kRegsSoftmax)
    return cudaErrorInvalidConfiguration;
  const int grid = min(p.n_items, sm_count());
  k_forward<D, BKV, kLinear><<<grid, kThreads, C::SMEM, st>>>(tmQ, tmK, tmV, tmKb, tmVs, tmHb, tmO,
                                                                p);
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
  // the per-block first-order mode is its own instantiation, so that the other modes'
  // kernels carry none of its code (registers)
  if (a.mode == BSA_MODE_PISA_BLOCK) {
    if (s.d == 64 && s.block == 64) return fwdtc::run<64, 64, true>(a, flag, kb16, vs16, hb16, st);
    if (s.d == 64 && s.block == 128) return fwdtc::run<64, 128, true>(a, flag, kb16, vs16, hb16, st);
    if (s.d == 128 && s.block == 64) return fwdtc::run<128, 64, true>(a, flag, kb16, vs16, hb16, st);
    return fwdtc::run<128, 128, true>(a, flag, kb16, vs16, hb16, st);
  }
  // head dim 64: the kernel whose row softmax is shared by a pair of threads
  // (forward_pair.cu), which measured faster there; head dim 128: the kernel here
  if (s.d == 64) return launch_forward_pair(a, flag, kb16, vs16, hb16, (int)Mp, st);
  if (s.block == 64) return fwdtc::run<128, 64, false>(a, flag, kb16, vs16, hb16, st);
  return fwdtc::run<128, 128, false>(a, flag, kb16, vs16, hb16, st);
}

}  // namespace bsa
