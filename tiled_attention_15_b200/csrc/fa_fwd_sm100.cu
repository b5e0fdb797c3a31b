// fa_fwd_sm100.cu -- fused, tiled attention forward pass (FlashAttention) for B200 / sm_100a.
//
// What is computed (mooersco.com article "昇腾CANN ops-transformer 仓的 FlashAttention
// 算子", section "昇腾NPU上的分块策略", steps 1-5): for every query row block and
// every key/value column block, S = Q K^T on the matrix unit, an online-softmax
// update of the running row maximum m and row sum l on the vector unit, and
// O += P V back on the matrix unit, with S and P kept on chip.  The B200 mapping:
//
//   * one persistent CTA per SM walks a list of work tiles; a work tile is
//     NQ = 2 query tiles of 128 rows (NQ = 1 for head_dim 256) of one
//     (batch, head);
//   * warp 9 (one thread) streams Q once per tile and K_j / V_j blocks of 128
//     keys through an NST-stage shared-memory ring with TMA (the page's double
//     buffering, deeper);
//   * warp 8 (one thread) issues tcgen05.mma: S_q = Q_q K_j^T into tensor memory
//     (fp32), then O_q += P_q V_j with P read from tensor memory, where the
//     softmax wrote it over S_q as 16-bit values;
//   * warps 0-3 and 4-7 are two softmax warpgroups, one per query tile, one row
//     per thread: row max, exp2 with the scale folded in, row sum, P back to
//     tensor memory; the partial O in tensor memory is rescaled only when the
//     row maximum grew by more than 2^8 since the last rescale (exact: any
//     common stabiliser gives the same softmax), and 1/l is applied once, in
//     the epilogue, which also writes the natural-log row LSE;
//   * causal attention skips key blocks above the diagonal and masks only the
//     blocks that straddle it (or the key tail);
//   * with NQ = 2 the two query tiles ping-pong: the tensor core works on one
//     tile's S or PV while the other tile's softmax runs;
//   * the epilogue writes O row by row in 16-byte pieces, or (fp16 launches
//     without a mask over at most 4096 keys: the STG instantiation) through a
//     4 KB shared-memory stage per softmax warp as whole 128-byte lines.
//
// Tensor memory (512 columns x 128 lanes x 32 bit): S_0 at column 0, S_1 at
// 128 (for NQ = 1 these are two S buffers of the single tile, used for
// alternate key blocks), O_q at 256 + q*D.
//
// Every wait on an mbarrier is bounded (kWaitLimitNs); a wait that runs out
// records FA_ERR_DEVICE_TIMEOUT in a device status word, makes the whole CTA
// leave its loops, waits (bounded) for its own TMA loads in flight, frees its
// tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "fa.h"
#include "sm100_ptx.cuh"

namespace fa {

__device__ unsigned int g_status = 0;
// Where the first timed-out wait was: CTA << 48 | warp << 40 | barrier shared address << 8 | parity.
__device__ unsigned long long g_timeout_site = 0;

constexpr int kBM = 128;  // query rows per query tile (MMA M)
constexpr int kBN = 128;  // keys per key/value block (MMA N of S, K of PV)
constexpr int kThreads = 384;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s: far above any legitimate wait
constexpr float kRescaleThreshold = 8.0f;         // log2 units: P <= 2^8 between rescales
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;
constexpr int kTileRing = 4;  // units the TMA thread may hand out ahead of the consumers

template <int D, int NQ, bool BIAS = false>
struct Geometry {
  static constexpr int DCH = D / 64;  // 128-byte (64-element) column chunks per row
  static constexpr int Q_BYTES = kBM * D * 2;
  static constexpr int KV_BYTES = kBN * D * 2;
  static constexpr int CHUNK_Q = kBM * 128;   // one 64-column chunk of a Q tile
  static constexpr int CHUNK_KV = kBN * 128;  // one 64-column chunk of a K/V block
  // K/V stages: what the shared memory left by the Q tiles holds (one query
  // tile leaves room for deeper staging, which decode-like launches need)
  // (score bias with two query tiles: one bias tile per query tile, 3 K/V stages at D = 128)
  static constexpr int NST = BIAS ? (NQ == 2 ? (D == 64 ? 8 : 3) : (D == 64 ? 8 : (D == 128 ? 4 : 2)))
                                  : NQ == 2 ? (D == 64 ? 8 : 4) : (D == 64 ? 12 : (D == 128 ? 6 : 2));
  // score-bias tiles: [2 boxes][128 rows][64 keys], 16-bit; one query tile: a
  // ring of NBS, two query tiles: one per query tile
  static constexpr int NBS = BIAS ? (D == 256 ? 1 : 2) : 0;
  static constexpr int BIAS_BYTES = 128 * 128 * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = NQ * Q_BYTES;
  static constexpr int OFF_BIAS = OFF_KV + NST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_BIAS + NBS * BIAS_BYTES;
  // mbarrier indices
  static constexpr int B_QFULL = 0, B_QEMPTY = 2, B_KVFULL = 4, B_KVEMPTY = 4 + NST,
                       B_SFULL = 4 + 2 * NST, B_PFULL = B_SFULL + 2, B_OFULL = B_PFULL + 2,
                       B_OEMPTY = B_OFULL + 2, B_PVDONE = B_OEMPTY + 2, B_TFULL = B_PVDONE + 1,
                       B_TEMPTY = B_TFULL + kTileRing, B_BFULL = B_TEMPTY + kTileRing,
                       B_BEMPTY = B_BFULL + NBS, B_MSTORED = B_BEMPTY + NBS,
                       B_MLAST = B_MSTORED + 2, NBAR = B_MLAST + 2;
  // tmem base (u32), abort flag (u32), then the ring of unit indices (kTileRing x s32)
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // ... then this CTA's stream-K unit range (2 x s32), then per query tile the
  // split-merge verdict (2 x s32: 1 = this CTA merges the tile)
  static constexpr int SMEM_BYTES = OFF_MISC + 8 + 4 * kTileRing + 8 + 8 + 1024;  // + alignment slack
  // The staged epilogue (two query tiles, no score bias; an instantiation of its
  // own) adds per softmax warp a 4 KB area, 32 rows x 64 columns of 16-bit output,
  // after everything else.  (Not in every kernel: with it a CTA takes the largest
  // shared-memory carveout, which leaves the L1 cache half the room.)
  static constexpr int OFF_STAGE = (OFF_MISC + 8 + 4 * kTileRing + 8 + 8 + 1023) & ~1023;
  static constexpr int SMEM_BYTES_STAGED = OFF_STAGE + 8 * 4096 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(NQ == 1 || BIAS || SMEM_BYTES_STAGED <= 232448, "shared memory budget (staged)");
  static_assert(NQ == 2 ? (256 + 2 * D <= 512) : (256 + D <= 512), "tensor memory budget");
};

struct FwdParams {
  void* o;
  float* lse;
  int B, Hq, Hkv, Nq, Nk, group;
  int causal;
  // Key window: query i sees keys i - wl .. i + wr; -1 is no bound.  wr is 0
  // for causal launches.  Windowed launches (wl >= 0, or wr >= 0 without
  // causal) use one query tile per work tile and are not split.  (Two fields,
  // not a third flag: a larger parameter block made the two-tile kernels spill.)
  int wl, wr;
  float c;          // scale * log2(e)
  int qt_per_head;  // work tiles per (batch, head)
  int n_tiles;
  int nkb;  // key blocks: ceil(Nk / kBN)
  // Split tiles: tiles [n_whole, n_tiles) are each processed as nsplit units, one
  // per part of the key blocks; n_units = n_whole + nsplit * (n_tiles - n_whole).
  // Each part leaves its un-normalised partial in the workspace and the last one
  // to finish a row group merges (see merge_epilogue).
  int n_whole, n_units, nsplit;
  int ws_rows;      // partial rows stored per split unit: the rows of the tile that
                    // exist, rounded up to whole warps (multiple of 32)
  // GQA packing (pack_g > 1): a work tile holds all pack_g query heads of one
  // key/value head, row r = (head r / Nq, query r % Nq), pack_g * Nq <= 128.
  int pack_g;
  // partial O (fp32), [partial][ws_rows / 32][D / 4][32 lanes] float4: one warp's
  // 32 rows interleaved by column quad, so that a warp's stores and loads of a
  // column quad are one contiguous 512-byte run; a tile's parts are consecutive
  float4* ws_o;
  float4* ws_ml;    // [partial][ws_rows] (m, l, l_rounded, 0)
  int* ws_cnt;      // [split tile][NQ][4 row groups] arrival counters (left at 0); one
                    // query tile per work tile uses [split tile][0][0] only
  // Dynamic schedule (with a workspace): sched[0] hands out units beyond the
  // first gridDim.x, sched[1] counts finished CTAs; the last CTA resets both.
  int* sched;
  // Stream-K (sk_w > 0; non-causal launches with fewer tiles than CTAs): the
  // sk_w = n_tiles * nkb key blocks of all tiles, flattened tile-major, are cut
  // into gridDim.x equal contiguous ranges, one per CTA.  CTA c runs one unit
  // per tile t that its range touches, with unit id c + t; the id also indexes
  // the unit's partial in the workspace (ids grow with (t, c), never repeat).
  // The host keeps sk_w * gridDim.x below 2^31.  The TMA thread publishes
  // these units through the unit ring, like the dynamic schedule's.
  int sk_w;
  int use_ring;  // units come through the shared-memory ring (sched or sk_w)
};

struct Tile {
  int bh;     // b * Hq + hq
  int row0;   // first query row of the work tile
  int kvz;    // b * Hkv + kv head
  int nblk[2];
  int j0[2];  // key windows, two query tiles: query tile q uses blocks j0[q] .. j0[q] + nblk[q] - 1
  int nb;
  int jb;     // first key block of this unit
  int slot;    // split-tile index, or -1 for a whole tile
  int part;    // which key part of a split tile
  int nparts;  // key parts of this split tile
  int store0;  // workspace index of part 0 (parts are stored consecutively)
};

template <int NQ, bool WIN = false>
__device__ __forceinline__ Tile get_tile(const FwdParams& p, int u) {
  Tile T;
  int t = u;
  int kb0 = 0, kb1 = p.nkb;  // split units: non-causal only (the host guarantees it)
  T.slot = -1;
  T.part = 0;
  T.nparts = 1;
  T.store0 = 0;
  if (p.sk_w > 0) {  // stream-K: this CTA's share of tile t
    const int c = blockIdx.x, C = gridDim.x, W = p.sk_w, nkb = p.nkb;
    t = u - c;
    const int base = t * nkb;
    const int b0 = c * W / C, b1 = (c + 1) * W / C;
    kb0 = max(b0, base) - base;
    kb1 = min(b1, base + nkb) - base;
    // key block b belongs to CTA ((b + 1) * C - 1) / W
    const int cf = ((base + 1) * C - 1) / W, cl = ((base + nkb) * C - 1) / W;
    T.slot = t;
    T.part = c - cf;
    T.nparts = cl - cf + 1;
    T.store0 = cf + t;
  } else if (u >= p.n_whole) {  // one of nsplit equal key parts of a split tile
    const int v = u - p.n_whole;
    T.slot = v / p.nsplit;
    T.part = v - T.slot * p.nsplit;
    T.nparts = p.nsplit;
    T.store0 = T.slot * p.nsplit;
    t = p.n_whole + T.slot;
    kb0 = (T.part * p.nkb) / p.nsplit;
    kb1 = ((T.part + 1) * p.nkb) / p.nsplit;
  }
  int qt;
  if (p.pack_g > 1) {  // one tile per (batch, key/value head)
    qt = 0;
    T.kvz = t;
    T.bh = (t / p.Hkv) * p.Hq + (t % p.Hkv) * p.pack_g;  // first query head of the group
  } else {
    const int BH = p.B * p.Hq;
    if (p.causal) {  // heaviest (last) query tiles first
      qt = p.qt_per_head - 1 - t / BH;
      T.bh = t % BH;
    } else {  // tiles of one head adjacent: K/V of a head stay hot in L2
      T.bh = t / p.qt_per_head;
      qt = t % p.qt_per_head;
    }
    const int b = T.bh / p.Hq, hq = T.bh % p.Hq;
    T.kvz = b * p.Hkv + hq / p.group;
  }
  T.row0 = qt * NQ * kBM;
  const int rows = p.pack_g > 1 ? p.pack_g * p.Nq : p.Nq;  // rows of the (packed) tile space
  T.j0[0] = T.j0[1] = 0;
  if constexpr (WIN) {  // key windows, two query tiles: each its own range in the union
    int lo[2] = {0, 0}, hi[2] = {0, 0};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int rf = T.row0 + q * kBM;
      const int rl = min(rf + kBM - 1, p.Nq - 1);
      const int hk = p.wr >= 0 ? min(p.Nk - 1, rl + p.wr) : p.Nk - 1;
      const int lk = p.wl >= 0 ? max(0, rf - p.wl) : 0;
      lo[q] = min(lk / kBN, p.nkb - 1);
      hi[q] = max(lo[q], hk / kBN);  // at least one block (rows with no key: O = 0, LSE = -inf)
    }
    const bool two = T.row0 + kBM < rows;
    T.jb = lo[0];
    T.nb = (two ? hi[1] : hi[0]) - lo[0] + 1;
    T.nblk[0] = hi[0] - lo[0] + 1;
    T.nblk[1] = two ? hi[1] - lo[1] + 1 : 0;
    T.j0[1] = two ? lo[1] - lo[0] : 0;
    return T;
  }
  T.jb = kb0;
  T.nb = 0;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int rf = T.row0 + q * kBM;
    int n = 0;
    if (q < NQ && rf < rows) {
      n = kb1 - kb0;
      if (NQ == 1 && (p.wl >= 0 || (p.wr >= 0 && !p.causal))) {  // this tile's own block range, at least one block
        const int rl = min(rf + kBM - 1, p.Nq - 1);
        const int hi = p.wr >= 0 ? min(p.Nk - 1, rl + p.wr) : p.Nk - 1;
        const int lo = p.wl >= 0 ? max(0, rf - p.wl) : 0;
        const int b_lo = min(lo / kBN, p.nkb - 1);
        T.jb = b_lo;
        n = max(1, hi / kBN + 1 - b_lo);  // rows that see no key still get O = 0, LSE = -inf
      } else if (p.causal && p.pack_g <= 1) {
        const int rl = min(rf + kBM - 1, p.Nq - 1);
        n = min(p.nkb, rl / kBN + 1);
      }
    }
    T.nblk[q] = n;
    T.nb = max(T.nb, n);
  }
  return T;
}

// Where row r (0..127) of query tile q of a work tile goes: its flat output row
// ((b * Hq + hq) * Nq + position), its query position (for the causal mask) and
// whether it exists.
struct RowInfo {
  size_t out_row;
  int pos;
  bool live;
};
__device__ __forceinline__ RowInfo row_info(const FwdParams& p, const Tile& T, int q, int r) {
  RowInfo ri;
  const int tr = T.row0 + q * kBM + r;  // row in the tile space
  if (p.pack_g > 1) {
    const int h = tr / p.Nq;
    ri.pos = tr - h * p.Nq;
    ri.live = h < p.pack_g;
    ri.out_row = (static_cast<size_t>(T.bh) + (ri.live ? h : 0)) * p.Nq + ri.pos;
  } else {
    ri.pos = tr;
    ri.live = tr < p.Nq;
    ri.out_row = static_cast<size_t>(T.bh) * p.Nq + (ri.live ? tr : 0);
  }
  return ri;
}

// Work tiles of this CTA, in a zig-zag over rounds of gridDim.x tiles so that
// heavy-first causal lists spread evenly.
struct TileIter {
  int r, cta, G, n;
  __device__ TileIter(int n_tiles) : r(-1), cta(blockIdx.x), G(gridDim.x), n(n_tiles) {}
  __device__ bool next(int& t) {
    while (true) {
      ++r;
      if (r * G >= n) return false;
      const int pos = (r & 1) ? (G - 1 - cta) : cta;
      t = r * G + pos;
      if (t < n) return true;
    }
  }
};

struct Ctx {
  uint32_t sbase;  // 1024-aligned shared-memory base (shared address space)
  uint32_t tmem;   // tensor-memory base address
  volatile uint32_t* abort_flag;
  volatile int* ring;  // unit indices published by the TMA thread (dynamic schedule)
  __device__ uint32_t bar(int i, int off_bar) const { return sbase + off_bar + 8u * i; }
};

// Bounded wait on an mbarrier phase.  Returns false (and makes every other
// wait of the CTA return false) when the time limit is reached.  A wait that
// times out only stores a packed site word in the CTA's abort flag (first one
// wins); publish_abort() turns it into the device status word at teardown.
// This keeps each of the many inlined wait sites small.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity,
                                         volatile uint32_t* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      const uint32_t site = 0x80000000u | ((threadIdx.x >> 5) << 24) | ((bar & 0x3FFFFu) << 1) | parity;
      atomicCAS(const_cast<uint32_t*>(abort_flag), 0u, site);
      return false;
    }
  }
  return true;
}

// Thread 0 at teardown: record the CTA's timed-out wait (if any) in the device
// status word and, for the first CTA to do so, its site.
__device__ __forceinline__ void publish_abort(uint32_t flag) {
  if (flag == 0u) return;
  if (atomicCAS(&g_status, 0u, static_cast<unsigned>(FA_ERR_DEVICE_TIMEOUT)) == 0u)
    g_timeout_site = (static_cast<unsigned long long>(blockIdx.x) << 48) |
                     (static_cast<unsigned long long>((flag >> 24) & 0x3Fu) << 40) |
                     (static_cast<unsigned long long>((flag >> 1) & 0x3FFFFu) << 8) | (flag & 1u);
}

// Wait that ignores the abort flag, with its own short limit (used only to
// drain this CTA's own TMA loads on the abort path).
__device__ __forceinline__ void drain_bar(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > 100000000ull) return;
}

// Work units of a CTA.  Static schedule (no ring): the zig-zag TileIter.
// Dynamic schedule: the TMA thread takes unit blockIdx.x first, then
// gridDim.x + atomicAdd(sched[0], 1) each time (heaviest units have the lowest
// indices); stream-K: the TMA thread takes the CTA's fixed unit range.  Either
// way it publishes every index -- or -1 at the end -- in a shared-memory ring
// (t_full: written; t_empty: read by the MMA thread and every softmax warp, 4
// per query tile).
template <int D, int NQ, bool BIAS = false>
__device__ __forceinline__ bool produce_unit(const Ctx& cx, const FwdParams& p, TileIter& it,
                                             uint32_t& n, int& u) {
  if (!p.use_ring) return it.next(u);
  using G = Geometry<D, NQ, BIAS>;
  int end = p.n_units;
  if (p.sk_w > 0) {  // stream-K: this CTA's fixed range, left by the prologue after the ring
    const volatile int* sk = cx.ring + kTileRing;
    u = sk[0] + static_cast<int>(n);
    end = sk[1];
  } else {
    u = (n == 0) ? static_cast<int>(blockIdx.x) : static_cast<int>(gridDim.x) + atomicAdd(p.sched, 1);
  }
  const int k = n % kTileRing;
  if (n >= (uint32_t)kTileRing &&
      !wait_bar(cx.bar(G::B_TEMPTY + k, G::OFF_BAR), ((n / kTileRing) - 1) & 1u, cx.abort_flag))
    return false;
  const int pub = u < end ? u : -1;
  cx.ring[k] = pub;
  mbar_arrive(cx.bar(G::B_TFULL + k, G::OFF_BAR));  // release: the index is visible after the wait
  ++n;
  return pub >= 0;
}
// Consumer side; `lane` < 0 for the single MMA thread, else the softmax warp's lane.
template <int D, int NQ, bool BIAS = false>
__device__ __forceinline__ bool consume_unit(const Ctx& cx, const FwdParams& p, TileIter& it,
                                             uint32_t& n, int& u, int lane) {
  if (!p.use_ring) return it.next(u);
  using G = Geometry<D, NQ, BIAS>;
  const int k = n % kTileRing;
  bool ok = wait_bar(cx.bar(G::B_TFULL + k, G::OFF_BAR), (n / kTileRing) & 1u, cx.abort_flag);
  if (lane >= 0) ok = __all_sync(0xffffffffu, ok);
  if (!ok) return false;
  u = cx.ring[k];
  ++n;
  if (lane >= 0) __syncwarp();
  if (lane <= 0) mbar_arrive(cx.bar(G::B_TEMPTY + k, G::OFF_BAR));
  return u >= 0;
}

__device__ __forceinline__ uint32_t pack2(float a, float b, bool bf16) {
  if (bf16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

// ---------------------------------------------------------------- TMA producer
// Score-bias mode bits (bias launches): 1 = one bias row for every query
// (broadcast over queries), 2 = a bias per query head, 4 = a bias per batch.
constexpr int kBiasRowBcast = 1, kBiasPerHead = 2, kBiasPerBatch = 4;

template <int D, int NQ, bool BIAS = false, bool WIN = false>
__device__ __forceinline__ void role_load(const Ctx& cx, const FwdParams& p, const CUtensorMap* tq,
                                          const CUtensorMap* tq4, const CUtensorMap* tk,
                                          const CUtensorMap* tv, const CUtensorMap* tb,
                                          int bias_mode) {
  using G = Geometry<D, NQ, BIAS>;
  prefetch_tmap(p.pack_g > 1 ? tq4 : tq);
  prefetch_tmap(tk);
  prefetch_tmap(tv);
  const uint64_t pol_kv = policy_evict_last();
  const uint64_t pol_q = policy_evict_first();
  uint32_t kv_it = 0, qe_phase[2] = {0u, 0u}, q_issued[2] = {0u, 0u};
  bool ok = true;
  auto load_q = [&](const Tile& T, int q) -> bool {
    if (q_issued[q]) {
      if (!wait_bar(cx.bar(G::B_QEMPTY + q, G::OFF_BAR), qe_phase[q], cx.abort_flag)) return false;
      qe_phase[q] ^= 1u;
    }
    if (p.pack_g > 1) {  // all pack_g heads of the group: one box of pack_g * Nq rows
      mbar_arrive_expect_tx(cx.bar(G::B_QFULL + q, G::OFF_BAR), p.pack_g * p.Nq * 128 * G::DCH);
#pragma unroll
      for (int c = 0; c < G::DCH; ++c)
        tma_load_3d(cx.sbase + G::OFF_Q + q * G::Q_BYTES + c * G::CHUNK_Q, tq4,
                    cx.bar(G::B_QFULL + q, G::OFF_BAR), c * 64, 0, T.kvz, pol_q);
    } else {
      mbar_arrive_expect_tx(cx.bar(G::B_QFULL + q, G::OFF_BAR), G::Q_BYTES);
#pragma unroll
      for (int c = 0; c < G::DCH; ++c)
        tma_load_3d(cx.sbase + G::OFF_Q + q * G::Q_BYTES + c * G::CHUNK_Q, tq,
                    cx.bar(G::B_QFULL + q, G::OFF_BAR), c * 64, T.row0 + q * kBM, T.bh, pol_q);
    }
    ++q_issued[q];
    return true;
  };
  auto load_kv = [&](const Tile& T, const CUtensorMap* m, int j) -> bool {
    const int st = kv_it % G::NST;
    if (kv_it >= (uint32_t)G::NST) {
      if (!wait_bar(cx.bar(G::B_KVEMPTY + st, G::OFF_BAR), ((kv_it / G::NST) - 1) & 1u,
                    cx.abort_flag))
        return false;
    }
    mbar_arrive_expect_tx(cx.bar(G::B_KVFULL + st, G::OFF_BAR), G::KV_BYTES);
#pragma unroll
    for (int c = 0; c < G::DCH; ++c)
      tma_load_3d(cx.sbase + G::OFF_KV + st * G::KV_BYTES + c * G::CHUNK_KV, m,
                  cx.bar(G::B_KVFULL + st, G::OFF_BAR), c * 64, (T.jb + j) * kBN, T.kvz, pol_kv);
    ++kv_it;
    return true;
  };
  // Bias launches: the [128 query rows x 128 keys] bias tile of block j, as two
  // 64-key boxes with 128-byte swizzle (one row when broadcast over queries).
  uint32_t b_it = 0;
  auto load_bias = [&](const Tile& T, int j) -> bool {
    if constexpr (BIAS) {
      const int bs = b_it % G::NBS;
      if (b_it >= (uint32_t)G::NBS &&
          !wait_bar(cx.bar(G::B_BEMPTY + bs, G::OFF_BAR), ((b_it / G::NBS) - 1) & 1u, cx.abort_flag))
        return false;
      const int rows = (bias_mode & kBiasRowBcast) ? 1 : kBM;
      mbar_arrive_expect_tx(cx.bar(G::B_BFULL + bs, G::OFF_BAR), 2 * rows * 128);
      const int hq = T.bh % p.Hq, b = T.bh / p.Hq;
#pragma unroll
      for (int box = 0; box < 2; ++box)
        tma_load_4d(cx.sbase + G::OFF_BIAS + bs * G::BIAS_BYTES + box * (G::BIAS_BYTES / 2), tb,
                    cx.bar(G::B_BFULL + bs, G::OFF_BAR), (T.jb + j) * kBN + box * 64,
                    (bias_mode & kBiasRowBcast) ? 0 : T.row0, (bias_mode & kBiasPerHead) ? hq : 0,
                    (bias_mode & kBiasPerBatch) ? b : 0, pol_kv);
      ++b_it;
    }
    return true;
  };
  TileIter it(p.n_units);
  uint32_t n_units_seen = 0;
  int t;
  while (ok && produce_unit<D, NQ, BIAS>(cx, p, it, n_units_seen, t)) {
    const Tile T = get_tile<NQ, WIN>(p, t);
    // Q0, then K0 (the first S MMA of the tile needs only these), then Q1 -- each
    // Q tile waits only for the last S MMA that read its previous contents.
    // K/V block order matches the MMA warp's consumption order:
    //   NQ = 2: K0, V0, K1, V1, ...      NQ = 1: K0, K1, V0, K2, V1, ...
    if (T.nblk[0] > 0 && !load_q(T, 0)) { ok = false; break; }
    if (!load_kv(T, tk, 0)) { ok = false; break; }
    if (BIAS && NQ == 1 && !load_bias(T, 0)) { ok = false; break; }
    if (NQ == 2 && T.nblk[1] > 0 && !load_q(T, 1)) { ok = false; break; }
    for (int s = 1; s < 2 * T.nb && ok; ++s) {
      int j;
      bool is_k;
      if (NQ == 2) { j = s / 2; is_k = (s & 1) == 0; }   // s=1:V0 s=2:K1 s=3:V1 ...
      else {                                              // s=1:K1 s=2:V0 s=3:K2 ...
        if (s == 2 * T.nb - 1) { j = T.nb - 1; is_k = false; }
        else { is_k = (s & 1) == 1; j = is_k ? (s + 1) / 2 : s / 2 - 1; }
      }
      if (!load_kv(T, is_k ? tk : tv, j)) ok = false;
      if (BIAS && NQ == 1 && ok && is_k && !load_bias(T, j)) ok = false;
    }
  }
  if (!ok) {  // abort: let this CTA's own loads land before the CTA exits
    for (uint32_t n = (kv_it > (uint32_t)G::NST ? kv_it - G::NST : 0); n < kv_it; ++n)
      drain_bar(cx.bar(G::B_KVFULL + n % G::NST, G::OFF_BAR), (n / G::NST) & 1u);
    for (int q = 0; q < 2; ++q)
      if (q_issued[q]) drain_bar(cx.bar(G::B_QFULL + q, G::OFF_BAR), (q_issued[q] - 1) & 1u);
    if constexpr (BIAS)
      for (uint32_t n = (b_it > (uint32_t)G::NBS ? b_it - G::NBS : 0); n < b_it; ++n)
        drain_bar(cx.bar(G::B_BFULL + n % G::NBS, G::OFF_BAR), (n / G::NBS) & 1u);
  }
}

// ---------------------------------------------------------------- score-bias producer
// Two query tiles with a score bias: one thread of warp 10 streams, per key
// block, each query tile's [128 x 128] bias tile into that query tile's own
// buffer (two 64-key boxes, 128-byte swizzle; one row when the bias is
// broadcast over queries), as soon as the tile's softmax warps have read the
// previous block's.  It takes the units from the same schedule as the others.
template <int D, int NQ, bool BIAS, bool WIN>
__device__ __forceinline__ void role_bias_load(const Ctx& cx, const FwdParams& p, const CUtensorMap* tb,
                                               int bias_mode) {
  using G = Geometry<D, NQ, BIAS>;
  prefetch_tmap(tb);
  const uint64_t pol = policy_evict_last();
  uint32_t issued[2] = {0u, 0u};
  bool ok = true;
  TileIter it(p.n_units);
  uint32_t n_units_seen = 0;
  int t;
  while (ok && consume_unit<D, NQ, BIAS>(cx, p, it, n_units_seen, t, -1)) {
    const Tile T = get_tile<NQ, WIN>(p, t);
    const int hq = T.bh % p.Hq, b = T.bh / p.Hq;
    const int rows = (bias_mode & kBiasRowBcast) ? 1 : kBM;
    for (int j = 0; j < T.nb && ok; ++j) {
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (j >= T.nblk[q]) continue;
        if (issued[q] > 0 &&
            !wait_bar(cx.bar(G::B_BEMPTY + q, G::OFF_BAR), (issued[q] - 1) & 1u, cx.abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(cx.bar(G::B_BFULL + q, G::OFF_BAR), 2 * rows * 128);
#pragma unroll
        for (int box = 0; box < 2; ++box)
          tma_load_4d(cx.sbase + G::OFF_BIAS + q * G::BIAS_BYTES + box * (G::BIAS_BYTES / 2), tb,
                      cx.bar(G::B_BFULL + q, G::OFF_BAR), (T.jb + j) * kBN + box * 64,
                      (bias_mode & kBiasRowBcast) ? 0 : T.row0 + q * kBM,
                      (bias_mode & kBiasPerHead) ? hq : 0, (bias_mode & kBiasPerBatch) ? b : 0, pol);
        ++issued[q];
      }
    }
  }
  if (!ok)  // abort: let this thread's own loads land before the CTA exits
    for (int q = 0; q < 2; ++q)
      if (issued[q] > 0) drain_bar(cx.bar(G::B_BFULL + q, G::OFF_BAR), (issued[q] - 1) & 1u);
}

// ---------------------------------------------------------------- MMA issuer
template <int D, int NQ, bool BF16, bool BIAS = false, bool WIN = false>
__device__ __forceinline__ void role_mma(const Ctx& cx, const FwdParams& p) {
  using G = Geometry<D, NQ, BIAS>;
  constexpr uint32_t kIdS = idesc_f16(kBM, kBN, BF16, false);  // Q, K both K-major
  constexpr uint32_t kIdPV = idesc_f16(kBM, D, BF16, true);    // V is N(=D)-major
  uint32_t kv_it = 0, q_phase[2] = {0u, 0u}, p_phase[2] = {0u, 0u}, oe_phase[2] = {0u, 0u};
  bool o_pending[2] = {false, false};
  const uint32_t tm = cx.tmem;
  auto B = [&](int i) { return cx.bar(i, G::OFF_BAR); };

  auto consume = [&](int& st) -> bool {
    st = kv_it % G::NST;
    const bool r = wait_bar(B(G::B_KVFULL + st), (kv_it / G::NST) & 1u, cx.abort_flag);
    ++kv_it;
    tc_fence_after();
    return r;
  };
  // Shared-memory descriptors are built once; each MMA of a K-loop only adds a
  // constant byte offset (>> 4) to the start-address field.
  const uint64_t dq0 = sdesc_sw128(cx.sbase + G::OFF_Q, 16, 1024);
  const uint64_t dkv0 = sdesc_sw128(cx.sbase + G::OFF_KV, 16, 1024);
  const uint64_t dv0 = sdesc_sw128(cx.sbase + G::OFF_KV, G::CHUNK_KV, 1024);
  auto issue_S = [&](int qt, int sbuf, int st) {
    const uint64_t a0 = dq0 + static_cast<uint64_t>((qt * G::Q_BYTES) >> 4);
    const uint64_t b0 = dkv0 + static_cast<uint64_t>((st * G::KV_BYTES) >> 4);
    const uint32_t d = tm + sbuf * 128;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off_a = ((kk >> 2) * G::CHUNK_Q + (kk & 3) * 32) >> 4;
      const uint32_t off_b = ((kk >> 2) * G::CHUNK_KV + (kk & 3) * 32) >> 4;
      mma_ss(d, a0 + off_a, b0 + off_b, kIdS, kk > 0 ? 1u : 0u);
    }
  };
  auto issue_PV = [&](int ot, int sbuf, int st, bool acc) {
    const uint64_t b0 = dv0 + static_cast<uint64_t>((st * G::KV_BYTES) >> 4);
    const uint32_t d = tm + 256 + ot * D, a = tm + sbuf * 128;
#pragma unroll
    for (int kk = 0; kk < kBN / 16; ++kk)
      mma_ts(d, a + kk * 8, b0 + static_cast<uint64_t>((kk * 2048) >> 4), kIdPV,
             (acc || kk > 0) ? 1u : 0u);
  };
  // Before the first PV of a tile into O_q: the previous tile's epilogue must
  // have read O_q out of tensor memory.
  auto o_ready = [&](int q) -> bool {
    if (!o_pending[q]) return true;
    if (!wait_bar(B(G::B_OEMPTY + q), oe_phase[q], cx.abort_flag)) return false;
    oe_phase[q] ^= 1u;
    o_pending[q] = false;
    tc_fence_after();
    return true;
  };
  auto q_ready = [&](int q) -> bool {
    if (!wait_bar(B(G::B_QFULL + q), q_phase[q], cx.abort_flag)) return false;
    q_phase[q] ^= 1u;
    tc_fence_after();
    return true;
  };
  // P V of one key block, once the softmax has written P into S buffer sb
  auto pv_block = [&](int ot, int sb, int st, bool acc) -> bool {
    if (!wait_bar(B(G::B_PFULL + sb), p_phase[sb], cx.abort_flag)) return false;
    p_phase[sb] ^= 1u;
    tc_fence_after();
    issue_PV(ot, sb, st, acc);
    return true;
  };

  TileIter it(p.n_units);
  uint32_t n_units_seen = 0;
  int t;
  while (consume_unit<D, NQ, BIAS>(cx, p, it, n_units_seen, t, -1)) {
    const Tile T = get_tile<NQ, WIN>(p, t);
    const int nb = T.nb;
    int kst;
    if (!consume(kst)) return;
    if (NQ == 2 && WIN) {
      // key windows: the same stream, query tile q taking part in blocks
      // j0[q] <= j < j0[q] + nblk[q] of the unit (j0[0] = 0)
      const int s1 = T.j0[1], e0 = T.nblk[0], e1 = T.j0[1] + T.nblk[1];
      auto in1 = [&](int j) { return j >= s1 && j < e1; };
      if (e0 > 0) {
        if (!q_ready(0)) return;
        issue_S(0, 0, kst);
        mma_commit(B(G::B_SFULL + 0));
        if (e0 == 1) mma_commit(B(G::B_QEMPTY + 0));
      }
      if (in1(0)) {
        if (!q_ready(1)) return;
        issue_S(1, 1, kst);
        mma_commit(B(G::B_SFULL + 1));
        if (e1 == 1) mma_commit(B(G::B_QEMPTY + 1));
      }
      mma_commit(B(G::B_KVEMPTY + kst));
      for (int j = 0; j < nb; ++j) {
        int vst;
        if (!consume(vst)) return;
        if (j < e0) {
          if (j == 0 && !o_ready(0)) return;
          if (!pv_block(0, 0, vst, j > 0)) return;
          if (j == e0 - 1) { mma_commit(B(G::B_OFULL + 0)); o_pending[0] = true; }
        }
        int kst2 = -1;
        if (j + 1 < nb) {
          if (!consume(kst2)) return;
          if (j + 1 < e0) {
            issue_S(0, 0, kst2);
            mma_commit(B(G::B_SFULL + 0));
            if (j + 1 == e0 - 1) mma_commit(B(G::B_QEMPTY + 0));
          }
        }
        if (in1(j)) {
          if (j == s1 && !o_ready(1)) return;
          if (!pv_block(1, 1, vst, j > s1)) return;
          if (j == e1 - 1) { mma_commit(B(G::B_OFULL + 1)); o_pending[1] = true; }
        }
        mma_commit(B(G::B_KVEMPTY + vst));
        if (kst2 >= 0) {
          if (in1(j + 1)) {
            if (j + 1 == s1 && !q_ready(1)) return;
            issue_S(1, 1, kst2);
            mma_commit(B(G::B_SFULL + 1));
            if (j + 1 == e1 - 1) mma_commit(B(G::B_QEMPTY + 1));
          }
          mma_commit(B(G::B_KVEMPTY + kst2));
        }
      }
    } else if (NQ == 2) {
      // stream: S0(0) S1(0) | PV0(j) S0(j+1) PV1(j) S1(j+1) | ...
      // q_empty[q] is committed right after the last S MMA that reads Q_q.
      if (T.nblk[0] > 0) {
        if (!q_ready(0)) return;
        issue_S(0, 0, kst);
        mma_commit(B(G::B_SFULL + 0));
        if (T.nblk[0] == 1) mma_commit(B(G::B_QEMPTY + 0));
      }
      if (T.nblk[1] > 0) {
        if (!q_ready(1)) return;
        issue_S(1, 1, kst);
        mma_commit(B(G::B_SFULL + 1));
        if (T.nblk[1] == 1) mma_commit(B(G::B_QEMPTY + 1));
      }
      mma_commit(B(G::B_KVEMPTY + kst));
      for (int j = 0; j < nb; ++j) {
        int vst;
        if (!consume(vst)) return;
        if (j < T.nblk[0]) {
          if (j == 0 && !o_ready(0)) return;
          if (!pv_block(0, 0, vst, j > 0)) return;
          if (j == T.nblk[0] - 1) { mma_commit(B(G::B_OFULL + 0)); o_pending[0] = true; }
        }
        int kst2 = -1;
        if (j + 1 < nb) {
          if (!consume(kst2)) return;
          if (j + 1 < T.nblk[0]) {
            issue_S(0, 0, kst2);
            mma_commit(B(G::B_SFULL + 0));
            if (j + 1 == T.nblk[0] - 1) mma_commit(B(G::B_QEMPTY + 0));
          }
        }
        if (j < T.nblk[1]) {
          if (j == 0 && !o_ready(1)) return;
          if (!pv_block(1, 1, vst, j > 0)) return;
          if (j == T.nblk[1] - 1) { mma_commit(B(G::B_OFULL + 1)); o_pending[1] = true; }
        }
        mma_commit(B(G::B_KVEMPTY + vst));
        if (kst2 >= 0) {
          if (j + 1 < T.nblk[1]) {
            issue_S(1, 1, kst2);
            mma_commit(B(G::B_SFULL + 1));
            if (j + 1 == T.nblk[1] - 1) mma_commit(B(G::B_QEMPTY + 1));
          }
          mma_commit(B(G::B_KVEMPTY + kst2));
        }
      }
    } else {
      // one query tile, two S buffers: S(0) | S(j+1) PV(j) | ...
      if (!q_ready(0)) return;
      issue_S(0, 0, kst);
      mma_commit(B(G::B_SFULL + 0));
      mma_commit(B(G::B_KVEMPTY + kst));
      if (nb == 1) mma_commit(B(G::B_QEMPTY + 0));
      for (int j = 0; j < nb; ++j) {
        if (j + 1 < nb) {
          if (!consume(kst)) return;
          issue_S(0, (j + 1) & 1, kst);
          mma_commit(B(G::B_SFULL + ((j + 1) & 1)));
          mma_commit(B(G::B_KVEMPTY + kst));
          if (j + 1 == nb - 1) mma_commit(B(G::B_QEMPTY + 0));
        }
        int vst;
        if (!consume(vst)) return;
        if (j == 0 && !o_ready(0)) return;
        // P(j) lives in S buffer j & 1, and each buffer has its own p_full barrier:
        // S(j+1) is already issued here, so a fast softmax warp may finish block j+1
        // before a slow one finishes block j -- one barrier per buffer keeps their
        // arrivals apart (a warp can never get two blocks ahead: S(j+2) follows PV(j)).
        if (!pv_block(0, j & 1, vst, j > 0)) return;
        mma_commit(B(G::B_PVDONE));
        mma_commit(B(G::B_KVEMPTY + vst));
        if (j == nb - 1) { mma_commit(B(G::B_OFULL + 0)); o_pending[0] = true; }
      }
    }
  }
}

// Exps of these pairs (bit k: pair index % 8 == k) run on the FMA pipe; the
// rest on MUFU.  MUFU throughput (16 ex2 / clock / SM) alone would equal the
// tensor-core time of S and PV at head_dim 128.
#ifndef FA_EMU_PAIRS
#define FA_EMU_PAIRS 0x11u  // pairs 0 and 4 of every 8: 1/4 of the exps
#endif
constexpr uint32_t kEmuPairs = FA_EMU_PAIRS;

// Row max / min of 128 scores: four independent chains of two-input max (min).
// (A three-input max.f32 produced wrong maxima for masked rows in this kernel,
// so only the two-input form is used.)
__device__ __forceinline__ float row_max(const uint32_t* v) {
  float a0 = __uint_as_float(v[0]), a1 = __uint_as_float(v[1]), a2 = __uint_as_float(v[2]),
        a3 = __uint_as_float(v[3]);
#pragma unroll
  for (int i = 4; i < kBN; i += 4) {
    a0 = fmaxf(a0, __uint_as_float(v[i]));
    a1 = fmaxf(a1, __uint_as_float(v[i + 1]));
    a2 = fmaxf(a2, __uint_as_float(v[i + 2]));
    a3 = fmaxf(a3, __uint_as_float(v[i + 3]));
  }
  return fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
}
__device__ __forceinline__ float row_min(const uint32_t* v) {
  float a0 = __uint_as_float(v[0]), a1 = __uint_as_float(v[1]), a2 = __uint_as_float(v[2]),
        a3 = __uint_as_float(v[3]);
#pragma unroll
  for (int i = 4; i < kBN; i += 4) {
    a0 = fminf(a0, __uint_as_float(v[i]));
    a1 = fminf(a1, __uint_as_float(v[i + 1]));
    a2 = fminf(a2, __uint_as_float(v[i + 2]));
    a3 = fminf(a3, __uint_as_float(v[i + 3]));
  }
  return fminf(fminf(a0, a1), fminf(a2, a3));
}
// The two bf16 halves of a packed word, widened (exactly) to fp32.
__device__ __forceinline__ F2 unpack_bf16x2(uint32_t w) {
  return F2{__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)};
}

// Epilogue of one key part of a split tile (one query tile: KV-cache decode
// tiles often have a single row group).  Each warp of the query tile's
// warpgroup stores its un-normalised O rows (fp32), stabiliser m and sums l,
// l_r; once all four warps have stored (a bounded mbarrier handshake), warp 0
// bumps the tile's arrival counter.  The CTA that arrives last (the nparts-th)
// merges the tile with all four warps -- one 32-row group each, or, when the
// tile has fewer row groups than warps (KV-cache decode), column slices of
// them -- reading the parts in part order:
//   M = max_s m_s,  a_s = 2^(m_s - M),  L = sum_s a_s l_s,
//   O = sum_s a_s O_s / L,  LSE = (M + log2 L) ln 2,
// and resets the counter to 0 for the next call.  No part waits for another
// CTA, and the result does not depend on which part finished last.  The
// partial rows of a warp are stored interleaved by column quad (see
// FwdParams::ws_o), so every store and load of the partials is a coalesced
// 512-byte run.  Returns false if a handshake wait gave up (abort).
template <int D, int NQ, bool BF16, class G>
__device__ __forceinline__ bool merge_epilogue(const Ctx& cx, uint32_t& m_phase, const FwdParams& p,
                                               const Tile& T, int q, int sub, int lane, uint32_t ocol,
                                               float m, float l, float l_r) {
  const uint32_t b_stored = cx.bar(G::B_MSTORED + q, G::OFF_BAR), b_last = cx.bar(G::B_MLAST + q, G::OFF_BAR);
  volatile int* verdict = cx.ring + kTileRing + 2 + q;
  const int g0 = q * kBM + sub * 32;  // first row of this warp in the work tile
  const int rr = g0 + lane;
  // warp-uniform: the warp's rows lie within the stored (padded) rows of the unit
  const bool stored = g0 < p.ws_rows;
  auto mlx = [&](int part, int r) { return (static_cast<size_t>(T.store0) + part) * p.ws_rows + r; };
  auto ox = [&](int part, int gr, int c4) {  // gr: first row of a 32-row group
    return ((static_cast<size_t>(T.store0) + part) * p.ws_rows + gr) * (D / 4) + c4 * 32 + lane;
  };
  if (stored) p.ws_ml[mlx(T.part, rr)] = make_float4(m, l, l_r, 0.f);
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += 32) {
    uint32_t orr[32];
    tmem_ld_x32(ocol + c0, orr);  // warp-collective: every lane takes part
    if (stored) {
#pragma unroll
      for (int x = 0; x < 8; ++x)
        p.ws_o[ox(T.part, g0, c0 / 4 + x)] =
            make_float4(__uint_as_float(orr[4 * x]), __uint_as_float(orr[4 * x + 1]),
                        __uint_as_float(orr[4 * x + 2]), __uint_as_float(orr[4 * x + 3]));
    }
  }
  __threadfence();
  __syncwarp();
  // all four warps have stored -> warp 0 takes the tile's verdict -> all read it
  if (lane == 0) mbar_arrive(b_stored);
  bool ok = wait_bar(b_stored, m_phase, cx.abort_flag);
  if (!__all_sync(0xffffffffu, ok)) return false;
  int* cnt = p.ws_cnt + (T.slot * NQ + q) * 4;
  if (sub == 0) {
    int old = 0;
    if (lane == 0) {
      old = atomicAdd(cnt, 1);
      *verdict = old == T.nparts - 1 ? 1 : 0;
      mbar_arrive(b_last);
    }
  }
  ok = wait_bar(b_last, m_phase, cx.abort_flag);
  if (!__all_sync(0xffffffffu, ok)) return false;
  m_phase ^= 1u;
  const bool last = *verdict != 0;
  __syncwarp();
  if (!last) return true;  // a later part merges this tile
  __threadfence();
  // this warp's share: row group gsel, column quads [c4a, c4b)
  const int rows_q = min(p.ws_rows - q * kBM, kBM);  // stored rows of this query tile (x32)
  const int ng = rows_q > 0 ? rows_q / 32 : 0;         // its row groups (1..4)
  if (ng == 0) return true;
  const int per = 4 / ng;                              // warps per row group (ng = 3: 1)
  const int gsel = sub / per, slice = sub % per;
  if (gsel >= ng) return true;
  const int c4a = slice * (D / 4) / per, c4b = (slice + 1) * (D / 4) / per;
  const int gr = q * kBM + gsel * 32;
  const RowInfo ri = row_info(p, T, q, gsel * 32 + lane);
  // Parts are read four at a time with all their loads issued before use, so
  // a tile merged from many parts (stream-K) pays one memory latency per four.
  const int np = T.nparts;
  float M = -INFINITY;
  for (int s0 = 0; s0 < np; s0 += 4) {
    float mk[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) mk[k] = s0 + k < np ? __ldcg(p.ws_ml + mlx(s0 + k, gr + lane)).x : -INFINITY;
#pragma unroll
    for (int k = 0; k < 4; ++k) M = fmaxf(M, mk[k]);
  }
  float L = 0.f, Lr = 0.f;
  for (int s0 = 0; s0 < np; s0 += 4) {
    float4 mk[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      mk[k] = s0 + k < np ? __ldcg(p.ws_ml + mlx(s0 + k, gr + lane)) : make_float4(-INFINITY, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a = ex2(mk[k].x - M);
      L = fmaf(a, mk[k].y, L);
      Lr = fmaf(a, mk[k].z, Lr);
    }
  }
  const float inv = 1.f / (BF16 ? Lr : L);
  uint16_t* orow = reinterpret_cast<uint16_t*>(p.o) + ri.out_row * D;
#pragma unroll 1
  for (int c4 = c4a; c4 < c4b; c4 += 4) {  // 16 columns per pass
    float z[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) z[x] = 0.f;
    for (int s0 = 0; s0 < np; s0 += 4) {
      float sc[4];
      float4 u[4][4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const bool in = s0 + k < np;
        const int sk = in ? s0 + k : s0;  // (a valid address; its weight is 0)
        sc[k] = in ? ex2(__ldcg(p.ws_ml + mlx(sk, gr + lane)).x - M) * inv : 0.f;
#pragma unroll
        for (int x = 0; x < 4; ++x) u[k][x] = __ldcg(p.ws_o + ox(sk, gr, c4 + x));
      }
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          z[4 * x] = fmaf(u[k][x].x, sc[k], z[4 * x]);
          z[4 * x + 1] = fmaf(u[k][x].y, sc[k], z[4 * x + 1]);
          z[4 * x + 2] = fmaf(u[k][x].z, sc[k], z[4 * x + 2]);
          z[4 * x + 3] = fmaf(u[k][x].w, sc[k], z[4 * x + 3]);
        }
    }
    if (ri.live) {
      uint4* dst = reinterpret_cast<uint4*>(orow + c4 * 4);
#pragma unroll
      for (int x = 0; x < 2; ++x)
        dst[x] = make_uint4(pack2(z[8 * x], z[8 * x + 1], BF16), pack2(z[8 * x + 2], z[8 * x + 3], BF16),
                            pack2(z[8 * x + 4], z[8 * x + 5], BF16),
                            pack2(z[8 * x + 6], z[8 * x + 7], BF16));
    }
  }
  if (slice == 0 && p.lse != nullptr && ri.live) p.lse[ri.out_row] = (M + log2f(L)) * kLn2;
  __syncwarp();
  if (sub == 0 && lane == 0) *cnt = 0;  // every part has arrived: safe to reset
  return true;
}

// Epilogue of one key part of a split tile, for the 32 rows of this warp (two
// query tiles: each query tile has four row groups, one per warp).  Each
// part stores its un-normalised O rows (fp32), its stabiliser m and sums l, l_r;
// then the warp bumps the counter of its row group.  The warp that arrives last
// (the nparts-th) reads all parts, in part order, and writes the merged rows:
//   M = max_s m_s,  a_s = 2^(m_s - M),  L = sum_s a_s l_s,
//   O = sum_s a_s O_s / L,  LSE = (M + log2 L) ln 2,
// then resets the counter to 0 for the next call.  No part waits for another,
// so no cross-CTA wait exists, and the result does not depend on which part
// finished last.  The partial rows of a warp are stored interleaved by column
// quad (see FwdParams::ws_o), so every store and load of the partials is a
// coalesced 512-byte run, and the merge keeps 8 loads per part in flight.
template <int D, int NQ, bool BF16>
__device__ __forceinline__ void merge_epilogue_rows(const FwdParams& p, const Tile& T, int q, int sub,
                                                    int lane, const RowInfo& ri, uint32_t ocol,
                                                    float m, float l, float l_r) {
  const int g0 = q * kBM + sub * 32;  // first row of this warp in the work tile
  const int rr = g0 + lane;
  // warp-uniform: the warp's rows lie within the stored (padded) rows of the unit
  const bool stored = g0 < p.ws_rows;
  auto mlx = [&](int part) { return (static_cast<size_t>(T.store0) + part) * p.ws_rows + rr; };
  auto ox = [&](int part, int c4) {
    return ((static_cast<size_t>(T.store0) + part) * p.ws_rows + g0) * (D / 4) + c4 * 32 + lane;
  };
  if (stored) p.ws_ml[mlx(T.part)] = make_float4(m, l, l_r, 0.f);
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += 32) {
    uint32_t orr[32];
    tmem_ld_x32(ocol + c0, orr);  // warp-collective: every lane takes part
    if (stored) {
#pragma unroll
      for (int x = 0; x < 8; ++x)
        p.ws_o[ox(T.part, c0 / 4 + x)] =
            make_float4(__uint_as_float(orr[4 * x]), __uint_as_float(orr[4 * x + 1]),
                        __uint_as_float(orr[4 * x + 2]), __uint_as_float(orr[4 * x + 3]));
    }
  }
  __threadfence();
  __syncwarp();
  int* cnt = p.ws_cnt + (T.slot * NQ + q) * 4 + sub;
  int old = 0;
  if (lane == 0) old = atomicAdd(cnt, 1);
  old = __shfl_sync(0xffffffffu, old, 0);
  if (old != T.nparts - 1) return;  // a later part merges these rows
  __threadfence();
  if (stored) {
    float M = -INFINITY;
    for (int s = 0; s < T.nparts; ++s) M = fmaxf(M, __ldcg(p.ws_ml + mlx(s)).x);
    float L = 0.f, Lr = 0.f;
    for (int s = 0; s < T.nparts; ++s) {
      const float4 ml = __ldcg(p.ws_ml + mlx(s));
      const float a = ex2(ml.x - M);
      L = fmaf(a, ml.y, L);
      Lr = fmaf(a, ml.z, Lr);
    }
    // a part in which a score bias removed every key of the row has m = -inf
    // (weight 0); a row with no key in any part has no softmax: O = 0, LSE = -inf
    const bool empty = M == -INFINITY;
    const float inv = empty ? 0.f : 1.f / (BF16 ? Lr : L);
    uint16_t* orow = reinterpret_cast<uint16_t*>(p.o) + ri.out_row * D;
#pragma unroll 1
    for (int c4 = 0; c4 < D / 4; c4 += 8) {  // 32 columns per pass
      float z[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) z[x] = 0.f;
      for (int s = 0; s < T.nparts; ++s) {
        const float sc = empty ? 0.f : ex2(__ldcg(p.ws_ml + mlx(s)).x - M) * inv;
        float4 u[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) u[x] = __ldcg(p.ws_o + ox(s, c4 + x));
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          z[4 * x] = fmaf(u[x].x, sc, z[4 * x]);
          z[4 * x + 1] = fmaf(u[x].y, sc, z[4 * x + 1]);
          z[4 * x + 2] = fmaf(u[x].z, sc, z[4 * x + 2]);
          z[4 * x + 3] = fmaf(u[x].w, sc, z[4 * x + 3]);
        }
      }
      if (ri.live) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c4 * 4);
#pragma unroll
        for (int x = 0; x < 4; ++x)
          dst[x] = make_uint4(pack2(z[8 * x], z[8 * x + 1], BF16), pack2(z[8 * x + 2], z[8 * x + 3], BF16),
                              pack2(z[8 * x + 4], z[8 * x + 5], BF16),
                              pack2(z[8 * x + 6], z[8 * x + 7], BF16));
      }
    }
    if (p.lse != nullptr && ri.live) p.lse[ri.out_row] = empty ? -INFINITY : (M + log2f(L)) * kLn2;
  }
  __syncwarp();
  if (lane == 0) *cnt = 0;
}

// ---------------------------------------------------------------- softmax + epilogue
template <int D, int NQ, bool BF16, bool BIAS = false, bool WIN = false, bool STG = false>
__device__ __forceinline__ void role_softmax(const Ctx& cx, const FwdParams& p, int wg, int sub,
                                             int lane, int bias_mode) {
  using G = Geometry<D, NQ, BIAS>;
  const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
  const uint32_t tm = cx.tmem + lane_off;
  auto B = [&](int i) { return cx.bar(i, G::OFF_BAR); };
  const float c = p.c;
  constexpr bool kWin = NQ == 1 || WIN;  // kernels that take key windows
  uint32_t s_phase[2] = {0u, 0u}, of_phase = 0u, pv_seen = 0u, m_phase = 0u;
  uint32_t b_cnt = 0, b_phase = 0u;  // bias tiles consumed; parity bit per stage
  const int q = (NQ == 2) ? wg : 0;

  TileIter it(p.n_units);
  uint32_t n_units_seen = 0;
  int t;
  while (consume_unit<D, NQ, BIAS>(cx, p, it, n_units_seen, t, lane)) {
    // Only what the key loop needs stays live across it; the epilogue decodes
    // the unit again (registers are the softmax warps' tightest resource).
    int nblk, rfirst, jb;
    {
      const Tile T0 = get_tile<NQ, WIN>(p, t);
      nblk = q ? T0.nblk[1] : T0.nblk[0];  // (selects keep the tile off the stack)
      rfirst = T0.row0 + q * kBM;
      jb = WIN ? T0.jb + (q ? T0.j0[1] : T0.j0[0]) : T0.jb;
    }
    if (nblk == 0) continue;
    // query position of this thread's row (causal mask; packing is non-causal only)
    const int row = rfirst + sub * 32 + lane;
    float m_used = -INFINITY, l = 0.f, l_r = 0.f;  // l: exact sum (LSE); l_r: rounded-P sum
    for (int j = 0; j < nblk; ++j) {
      const int sb = (NQ == 2) ? q : (j & 1);
      // (selects, not s_phase[sb]: a runtime index would put the array on the stack)
      bool ok = wait_bar(B(G::B_SFULL + sb), sb ? s_phase[1] : s_phase[0], cx.abort_flag);
      if (!__all_sync(0xffffffffu, ok)) return;
      if (sb) s_phase[1] ^= 1u;
      else s_phase[0] ^= 1u;
      tc_fence_after();
      uint32_t sr[kBN];
      tmem_ld_x128(tm + sb * 128, sr);

      const int kbase = (jb + j) * kBN;
      // (key windows exist in the one-query-tile kernels only; a score bias
      // enters the row max, so bias launches take the masked path every block)
      const bool masked =
          BIAS || (kWin ? (kbase + kBN > p.Nk) || (p.wr >= 0 && kbase + kBN - 1 > rfirst + p.wr) ||
                              (p.wl >= 0 && kbase < rfirst + kBM - 1 - p.wl)
                        : (kbase + kBN > p.Nk) || (p.causal && kbase + kBN - 1 > rfirst));
      float m_blk;
      bool raw = false;  // masked scores left unscaled (the scale enters with the exponent)
      if (masked) {  // -inf where the key is outside the window or past Nk (see each branch)
        int lim = p.Nk - kbase;  // keys [lo, lim) of the block are visible to this row
        if constexpr (BIAS) {
          // the tile holds this row's 128 bias values as 16 swizzled 16-byte
          // units (one row for every query when broadcast over queries)
          // keys of the block before lim are visible (one query tile: the key
          // window's right bound; its left bound is applied after the bias)
          if constexpr (kWin) {
            if (p.wr >= 0) lim = min(lim, row + p.wr - kbase + 1);
          } else if (p.causal) {
            lim = min(lim, row - kbase + 1);
          }
          const int bs = NQ == 2 ? q : static_cast<int>(b_cnt % G::NBS);
          ok = wait_bar(B(G::B_BFULL + bs), (b_phase >> bs) & 1u, cx.abort_flag);
          if (!__all_sync(0xffffffffu, ok)) return;
          b_phase ^= 1u << bs;
          ++b_cnt;
          const uint32_t brow = (bias_mode & kBiasRowBcast) ? 0u : static_cast<uint32_t>(sub * 32 + lane);
          const uint32_t bbase = cx.sbase + G::OFF_BIAS + bs * G::BIAS_BYTES + brow * 128u;
          // scale * s + bias in natural-log units, one packed multiply-add per two
          // keys (log2 e enters with the exponent's multiply-add); the key-range
          // test only where some lane's row ends inside the block
          const float sc_nat = c * (1.f / kLog2e);
          const bool all_visible = __all_sync(0xffffffffu, lim >= kBN);
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            uint32_t w[4];
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                         : "r"(bbase + (u >> 3) * (G::BIAS_BYTES / 2) +
                               ((static_cast<uint32_t>(u & 7) ^ (brow & 7u)) << 4)));
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = u * 8 + 2 * e;
              F2 bv;
              if (BF16) {
                bv = unpack_bf16x2(w[e]);
              } else {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
                bv = f2(f.x, f.y);
              }
              const F2 x = ffma2(f2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])),
                                 f2(sc_nat, sc_nat), bv);
              if (all_visible) {
                sr[i] = __float_as_uint(x.x);
                sr[i + 1] = __float_as_uint(x.y);
              } else {
                sr[i] = __float_as_uint(i < lim ? x.x : -INFINITY);
                sr[i + 1] = __float_as_uint(i + 1 < lim ? x.y : -INFINITY);
              }
            }
          }
          if constexpr (kWin) {  // left bound of a key window: keys before lo
            const int lo = p.wl >= 0 ? row - p.wl - kbase : 0;
            if (__any_sync(0xffffffffu, lo > 0)) {
#pragma unroll
              for (int i = 0; i < kBN; ++i)
                if (i < lo) sr[i] = __float_as_uint(-INFINITY);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(B(G::B_BEMPTY + bs));
        } else if (kWin) {
          if (p.wr >= 0) lim = min(lim, row + p.wr - kbase + 1);
          const int lo = p.wl >= 0 ? row - p.wl - kbase : 0;
          const uint32_t span = static_cast<uint32_t>(max(lim - lo, 0));
#pragma unroll
          for (int i = 0; i < kBN; ++i)
            sr[i] = __float_as_uint(static_cast<uint32_t>(i - lo) < span ? __uint_as_float(sr[i]) * c
                                                                          : -INFINITY);
        } else {
          if (p.causal) lim = min(lim, row - kbase + 1);
          // fp16: raw scores, -inf * sign(c) past the row (c enters with the
          // exponent; bf16 keeps the scaled form, which its register budget fits)
          if (!BF16 && c != 0.f) {
            raw = true;
            const uint32_t off = __float_as_uint(c > 0.f ? -INFINITY : INFINITY);
#pragma unroll
            for (int i = 0; i < kBN; ++i) sr[i] = (i < lim) ? sr[i] : off;
          } else {
#pragma unroll
            for (int i = 0; i < kBN; ++i)
              sr[i] = __float_as_uint((i < lim) ? __uint_as_float(sr[i]) * c : -INFINITY);
          }
        }
        if (raw) m_blk = (c > 0.f ? row_max(sr) : row_min(sr)) * c;
        else m_blk = row_max(sr) * (BIAS ? kLog2e : 1.f);  // (a bias: natural-log units)
      } else {  // max of raw scores; the scale (of either sign) is applied to the max
        m_blk = (c >= 0.f ? row_max(sr) : row_min(sr)) * c;
      }
      // stabiliser update (log2 units); rescale only when the max grew by > 2^8
      float alpha = 1.f;
      bool need = false;
      if (j == 0) {
        m_used = m_blk;
      } else if (m_blk > m_used + kRescaleThreshold) {
        alpha = ex2(m_used - m_blk);
        m_used = m_blk;
        need = true;
      }
      const float neg_m = (m_used == -INFINITY) ? 0.f : -m_used;
      const float cs = BIAS ? kLog2e : (masked && !raw) ? 1.f : c;
      // bf16 only: also sum the rounded P that the PV product actually uses, and
      // normalise O by that sum -- the weights then sum to one exactly, which
      // removes the bf16 rounding error of the dominant weight(s) from O.
      // P goes back to tensor memory (over S) in groups of 16 packed pairs as soon
      // as a group is ready, which keeps the live register set small.
      F2 acc[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
      F2 accr[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
      for (int g = 0; g < kBN / 32; ++g) {
        uint32_t pk[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int i = g * 16 + u;
          const F2 sv = f2(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]));
          // masked blocks hold already scaled scores (cs = 1); masked keys are -inf:
          // 0 from MUFU, ~2^-125 from the FMA-pipe exp2 (negligible against l >= 1)
          const F2 x = ffma2(sv, f2(cs, cs), f2(neg_m, neg_m));
          F2 pr;
          if ((kEmuPairs >> (i & 7)) & 1u) pr = exp2_fma2(x);  // FMA pipe
          else pr = f2(ex2(x.x), ex2(x.y));                   // MUFU
          acc[u & 3] = fadd2(acc[u & 3], pr);
          pk[u] = pack2(pr.x, pr.y, BF16);
          if (BF16) accr[u & 1] = fadd2(accr[u & 1], unpack_bf16x2(pk[u]));
        }
        tmem_st_x16(tm + sb * 128 + g * 16, pk);
      }
      const F2 a01 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
      l = l * alpha + (a01.x + a01.y);
      if (BF16) {
        const F2 r01 = fadd2(accr[0], accr[1]);
        l_r = l_r * alpha + (r01.x + r01.y);
      }
      if (__any_sync(0xffffffffu, need)) {
        if (NQ == 1) {  // PV(j-1) must have finished accumulating into O
          ok = wait_bar(B(G::B_PVDONE), (pv_seen + j - 1) & 1u, cx.abort_flag);
          if (!__all_sync(0xffffffffu, ok)) return;
          tc_fence_after();
        }
        const float a = need ? alpha : 1.f;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t orr[32];
          tmem_ld_x32(tm + 256 + q * D + c0, orr);
#pragma unroll
          for (int x = 0; x < 32; ++x) orr[x] = __float_as_uint(__uint_as_float(orr[x]) * a);
          tmem_st_x32(tm + 256 + q * D + c0, orr);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(B(G::B_PFULL + sb));
    }
    pv_seen += nblk;

    // epilogue: O = O_acc / l, rounded to the input dtype; LSE in natural log
    bool ok = wait_bar(B(G::B_OFULL + q), of_phase, cx.abort_flag);
    if (!__all_sync(0xffffffffu, ok)) return;
    of_phase ^= 1u;
    tc_fence_after();
    int t_again;  // opaque copy: the compiler must not keep the first decode live
    asm volatile("mov.b32 %0, %1;" : "=r"(t_again) : "r"(t));
    const Tile T = get_tile<NQ, WIN>(p, t_again);
    const RowInfo ri = row_info(p, T, q, sub * 32 + lane);
    const bool live = ri.live;
    const float m_sub = (m_used == -INFINITY) ? 0.f : m_used;
    if (T.slot >= 0) {
      if constexpr (NQ == 2) {
        merge_epilogue_rows<D, NQ, BF16>(p, T, q, sub, lane, ri, tm + 256 + q * D,
                                         BIAS ? m_used : m_sub, l, l_r);
      } else if (!merge_epilogue<D, NQ, BF16, G>(cx, m_phase, p, T, q, sub, lane, tm + 256 + q * D,
                                                 m_sub, l, l_r)) {
        return;
      }
    } else {
      // a row that saw no key (key windows, or a bias of -inf on every key) has no
      // softmax: O = 0, LSE = -inf
      const bool empty = (kWin || BIAS) && m_used == -INFINITY;
      const float inv_l = empty ? 0.f : 1.f / (BF16 ? l_r : l);
      if constexpr (STG) {
        // Each 64-column half goes through the warp's staging area: the thread's
        // own row in (16-byte units rotated by row, so neither direction has bank
        // conflicts), then each store instruction writes four whole 128-byte row
        // segments instead of 32 scattered 16-byte pieces.  (The staging address
        // is an opaque copy: hoisted out of the unit loop it would hold a
        // register through the key loop.)
        uint32_t stg;
        asm volatile("mov.b32 %0, %1;"
                     : "=r"(stg)
                     : "r"(cx.sbase + G::OFF_STAGE + static_cast<uint32_t>(wg * 4 + sub) * 4096u));
        const unsigned orow = live ? static_cast<unsigned>(ri.out_row) : 0xffffffffu;
        const uint32_t cu = static_cast<uint32_t>(lane & 7);
#pragma unroll 1
        for (int h = 0; h < D / 64; ++h) {
#pragma unroll 1
          for (int u0 = 0; u0 < 8; u0 += 4) {
            uint32_t orr[32];
            tmem_ld_x32(tm + 256 + q * D + h * 64 + u0 * 8, orr);
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
              const uint32_t u = static_cast<uint32_t>(u0 + uu);
              uint32_t w[4];
#pragma unroll
              for (int x = 0; x < 4; ++x)
                w[x] = pack2(__uint_as_float(orr[8 * uu + 2 * x]) * inv_l,
                             __uint_as_float(orr[8 * uu + 2 * x + 1]) * inv_l, BF16);
              st_shared_v4(stg + static_cast<uint32_t>(lane) * 128u + ((u ^ (lane & 7u)) << 4), w);
            }
          }
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t r = static_cast<uint32_t>(4 * k + (lane >> 3));
            uint32_t w[4];
            ld_shared_v4(stg + r * 128u + ((cu ^ (r & 7u)) << 4), w);
            const unsigned dst_row = __shfl_sync(0xffffffffu, orow, static_cast<int>(r));
            if (dst_row != 0xffffffffu)
              reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.o) +
                                       static_cast<size_t>(dst_row) * D + h * 64)[cu] =
                  make_uint4(w[0], w[1], w[2], w[3]);
          }
          __syncwarp();
        }
      } else {
      uint16_t* orow = reinterpret_cast<uint16_t*>(p.o) + ri.out_row * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t orr[32];
        tmem_ld_x32(tm + 256 + q * D + c0, orr);
        uint32_t w[16];
#pragma unroll
        for (int x = 0; x < 16; ++x)
          w[x] = pack2(__uint_as_float(orr[2 * x]) * inv_l, __uint_as_float(orr[2 * x + 1]) * inv_l,
                       BF16);
        if (live) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int x = 0; x < 4; ++x)
            dst[x] = make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
        }
      }
      }
      if (p.lse != nullptr && live)
        p.lse[ri.out_row] = empty ? -INFINITY : (m_sub + log2f(l)) * kLn2;
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(B(G::B_OEMPTY + q));
  }
}

template <int D, int NQ, bool BF16, bool BIAS = false, bool WIN = false, bool STG = false>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_q4,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const FwdParams p, const __grid_constant__ CUtensorMap tm_b, const int bias_mode) {
  using G = Geometry<D, NQ, BIAS>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  uint32_t* misc = reinterpret_cast<uint32_t*>(gbase + G::OFF_MISC);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  Ctx cx;
  cx.sbase = sbase;
  cx.abort_flag = misc + 1;
  cx.ring = reinterpret_cast<volatile int*>(misc + 2);
  if (threadIdx.x == 0) {
    auto B = [&](int i) { return cx.bar(i, G::OFF_BAR); };
    for (int q = 0; q < 2; ++q) {  // one pair per query tile: the next tile's Q0 loads early
      mbar_init(B(G::B_QFULL + q), 1);
      mbar_init(B(G::B_QEMPTY + q), 1);
    }
    for (int s = 0; s < G::NST; ++s) {
      mbar_init(B(G::B_KVFULL + s), 1);
      mbar_init(B(G::B_KVEMPTY + s), 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(B(G::B_SFULL + q), 1);
      mbar_init(B(G::B_PFULL + q), 4);
      mbar_init(B(G::B_OFULL + q), 1);
      mbar_init(B(G::B_OEMPTY + q), 4);
    }
    mbar_init(B(G::B_PVDONE), 1);
    for (int q = 0; q < 2; ++q) {
      mbar_init(B(G::B_MSTORED + q), 4);  // the four warps of query tile q's warpgroup
      mbar_init(B(G::B_MLAST + q), 1);
    }
    for (int k = 0; k < kTileRing; ++k) {
      mbar_init(B(G::B_TFULL + k), 1);
      // the MMA thread, the softmax warps (and the bias producer)
      mbar_init(B(G::B_TEMPTY + k), 1 + 4 * NQ + ((BIAS && NQ == 2) ? 1 : 0));
    }
    for (int k = 0; k < G::NBS; ++k) {
      mbar_init(B(G::B_BFULL + k), 1);
      mbar_init(B(G::B_BEMPTY + k), 4);  // the four softmax warps
    }
    misc[1] = 0u;
    if (p.sk_w > 0) {  // stream-K: the units c + t, t over the tiles this CTA's range touches
      const int c = blockIdx.x, C = gridDim.x, W = p.sk_w;
      int* sk = reinterpret_cast<int*>(misc + 2 + kTileRing);
      sk[0] = c + c * W / C / p.nkb;
      sk[1] = c + ((c + 1) * W / C - 1) / p.nkb + 1;
    }
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(misc), G::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cx.tmem = misc[0];

  // Registers: 168 per thread at launch (384 threads, one CTA per SM); the two
  // softmax warpgroups take kSoftmaxRegs, the MMA / TMA / idle warpgroup keeps
  // the rest (2 x 128 x 208 + 128 x 88 = 2 x 128 x 200 + 128 x 104 = 64512 =
  // 384 x 168). The two-query-tile kernel's MMA, TMA and bias-producer code
  // needs the 104 of the second split (with 88 it spills in its loops); bf16
  // with one query tile or a key window takes the first split, whose softmax
  // sums rounded P in registers that 200 do not hold without spilling.
  // The wait helpers are inlined: ptxas cannot allocate a call inside a region
  // resized this way.
  constexpr int kSoftmaxRegs = (BF16 && (NQ == 1 || WIN)) ? 208 : 200;
  constexpr int kOtherRegs = (384 * 168 - 256 * kSoftmaxRegs) / 128;
  if (warp < 8) setmaxnreg_inc<kSoftmaxRegs>();
  else setmaxnreg_dec<kOtherRegs>();
  if (warp < 8) {
    if (NQ == 2 || warp < 4)
      role_softmax<D, NQ, BF16, BIAS, WIN, STG>(cx, p, warp >> 2, warp & 3, lane, bias_mode);
  } else if (warp == 8) {
    if (lane == 0) role_mma<D, NQ, BF16, BIAS, WIN>(cx, p);
  } else if (warp == 9) {
    if (lane == 0) role_load<D, NQ, BIAS, WIN>(cx, p, &tm_q, &tm_q4, &tm_k, &tm_v, &tm_b, bias_mode);
  } else if (warp == 10) {
    if (BIAS && NQ == 2 && lane == 0) role_bias_load<D, NQ, BIAS, WIN>(cx, p, &tm_b, bias_mode);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) publish_abort(*cx.abort_flag);
  if (threadIdx.x == 0 && p.sched != nullptr) {  // the last CTA to finish resets the schedule
    __threadfence();
    if (atomicAdd(p.sched + 1, 1) == static_cast<int>(gridDim.x) - 1) {
      p.sched[0] = 0;
      p.sched[1] = 0;
      __threadfence();
    }
  }
  if (warp == 8) {
    if (*cx.abort_flag) {  // abort path: give issued MMAs time to retire before freeing TMEM
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 2000000ull) {
      }
    }
    tmem_dealloc(cx.tmem, G::TMEM_COLS);
  }
}

// Runs the kernels' bounded wait on an mbarrier that nothing arrives on: after the
// time limit it records FA_ERR_DEVICE_TIMEOUT and the site, and returns (tests the
// failure detection without hanging or faulting the device).
__global__ void wait_timeout_probe_kernel() {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0u;
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    wait_bar(smem_u32(&bar), 0u, &abort_flag);
    publish_abort(abort_flag);
  }
}

// Evaluates the FMA-pipe exp2 used by the softmax on an array (diagnostics / tests).
__global__ void exp2_fma_eval_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const F2 r = exp2_fma2(f2(x[i], x[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_fma2(f2(x[i], 0.f)).x;
  }
}

}  // namespace fa

// ============================================================================ host side
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

constexpr int kMaxDevices = 64;
// Longest key range that takes the staged epilogue (32 key blocks): past it the
// epilogue is a small share of a tile and the larger shared-memory footprint
// costs more than the whole-line stores save.
constexpr int kStagedMaxKeys = 32 * fa::kBN;
struct DeviceState {
  std::once_flag once;
  int sms = 0;
  bool sm100 = false;
};
DeviceState g_dev[kMaxDevices];

// 3-D map over a [Z][rows][D] 16-bit tensor: box = 64 columns x box_rows rows x 1,
// 128-byte swizzle (the layout the tcgen05 shared-memory descriptors describe).
bool make_map(CUtensorMap* m, const void* ptr, int D, long long rows, long long Z, int box_rows,
              bool bf16) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)Z};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  const cuuint32_t box[3] = {64u, (cuuint32_t)box_rows, 1u};
  const cuuint32_t es[3] = {1u, 1u, 1u};
  const CUresult r =
      enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
          const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int nq_for(int D) { return D == 256 ? 1 : 2; }

// GQA packing: when the query heads of one key/value head fit one 128-row tile
// together (decode-like shapes), one work tile holds all of them.
bool pack_heads(int Hq, int Hkv, int Nq, int causal) {
  const int g = Hq / Hkv;
  return g > 1 && !causal && static_cast<long long>(g) * Nq <= fa::kBM;
}

std::atomic<int> g_max_ctas{0};

// Workspace partition for split tails.  The arrival counters come first, at a
// fixed place whatever the call (they must stay zero between calls); the
// partial results of up to max_split tiles follow.  Offsets are multiples of
// 256 bytes.
constexpr int kMaxSplit = 1024;  // >= half the SMs of any device
constexpr int kMinSplitBlocks = 8;
constexpr int kMinPartBlocks = 4;  // least key blocks per CTA under stream-K
struct WsLayout {
  size_t cnt_off, ml_off, o_off, total;
};
// Partial results: n_split tiles x nsplit parts x rows per tile.
WsLayout ws_layout(int D, int rows, int n_split, int nsplit) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  WsLayout L;
  L.cnt_off = 0;  // split counters, then the two schedule counters
  L.ml_off = up(static_cast<size_t>(kMaxSplit) * 2 * 4 * sizeof(int) + 2 * sizeof(int));
  const size_t units = static_cast<size_t>(n_split) * nsplit * rows;
  L.o_off = L.ml_off + up(units * sizeof(float4));
  L.total = L.o_off + up(units * D * sizeof(float));
  return L;
}

// Scratch modes of a launch: a caller workspace (split only if it fits), or the
// library's static scratch (a split that does not fit is an error, and the
// arrival counters are cleared on the stream before the kernel).
enum class Scratch { kCaller, kStatic };

// A score bias [B][H][Nq][Nk] (16-bit, keys contiguous) given by element strides;
// a zero stride broadcasts that dimension.
struct BiasArg {
  const void* ptr;
  long long sb, sh, sq;
};

// 4-D map over the bias with 64-key x `rows`-query boxes, 128-byte swizzle; a
// broadcast dimension has extent 1 (its coordinate is always 0).
bool make_bias_map(CUtensorMap* m, const BiasArg& a, int B, int H, int Nq, int Nk, bool bf16) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)Nk, (cuuint64_t)(a.sq ? Nq : 1), (cuuint64_t)(a.sh ? H : 1),
                              (cuuint64_t)(a.sb ? B : 1)};
  // strides of extent-1 dimensions are never used; keep them valid and increasing
  const cuuint64_t s1 = a.sq ? (cuuint64_t)a.sq * 2 : (cuuint64_t)((Nk * 2 + 15) / 16 * 16);
  const cuuint64_t s2 = a.sh ? (cuuint64_t)a.sh * 2 : s1 * dims[1];
  const cuuint64_t s3 = a.sb ? (cuuint64_t)a.sb * 2 : s2 * dims[2];
  const cuuint64_t strides[3] = {s1, s2, s3};
  const cuuint32_t box[4] = {64u, a.sq ? 128u : 1u, 1u, 1u};
  const cuuint32_t es[4] = {1u, 1u, 1u, 1u};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
             const_cast<void*>(a.ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int NQ, bool BF16, bool BIAS = false, bool WIN = false, bool STG = false>
int launch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
           int Hkv, int Nq, int Nk, float scale, int causal, int wl, int wr, cudaStream_t stream,
           int dev, void* ws, size_t ws_bytes, Scratch mode, const BiasArg* bias = nullptr) {
  using G = fa::Geometry<D, NQ, BIAS>;
  static_assert(!STG || (NQ == 2 && !BIAS), "the staged epilogue: two query tiles, no bias");
  constexpr int kSmem = STG ? G::SMEM_BYTES_STAGED : G::SMEM_BYTES;
  static bool attr_done[kMaxDevices] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (!attr_done[dev]) {
      if (cudaFuncSetAttribute(fa::fa_fwd_kernel<D, NQ, BF16, BIAS, WIN, STG>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess)
        return FA_ERR_LAUNCH;
      attr_done[dev] = true;
    }
  }
  const int g = Hq / Hkv;
  const bool windowed = wl >= 0 || wr >= 0;
  const bool pack = !BIAS && !windowed && pack_heads(Hq, Hkv, Nq, causal);
  CUtensorMap tq, tq4, tk, tv;
  if (!make_map(&tq, q, D, Nq, (long long)B * Hq, fa::kBM, BF16) ||
      !make_map(&tk, k, D, Nk, (long long)B * Hkv, fa::kBN, BF16) ||
      !make_map(&tv, v, D, Nk, (long long)B * Hkv, fa::kBN, BF16))
    return FA_ERR_DRIVER;
  if (pack) {  // q viewed as [B*Hkv][g*Nq][D]: a group's query rows are contiguous
    if (!make_map(&tq4, q, D, (long long)g * Nq, (long long)B * Hkv, g * Nq, BF16))
      return FA_ERR_DRIVER;
  } else {
    tq4 = tq;
  }
  fa::FwdParams p;
  p.o = o;
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.group = g;
  p.causal = causal ? 1 : 0;
  p.wl = wl;
  p.wr = causal ? 0 : wr;
  p.c = scale * 1.4426950408889634f;
  p.pack_g = pack ? g : 1;
  p.qt_per_head = pack ? 1 : (Nq + NQ * fa::kBM - 1) / (NQ * fa::kBM);
  p.n_tiles = pack ? B * Hkv : B * Hq * p.qt_per_head;
  p.nkb = (Nk + fa::kBN - 1) / fa::kBN;
  int ctas = g_dev[dev].sms;
  const int cap = g_max_ctas.load();
  if (cap > 0 && cap < ctas) ctas = cap;
  // rows of a work tile that exist, rounded up to whole warps (partials are
  // stored for these only)
  p.ws_rows = pack ? g * Nq : (p.qt_per_head == 1 ? (Nq < NQ * fa::kBM ? Nq : NQ * fa::kBM)
                                                   : NQ * fa::kBM);
  p.ws_rows = (p.ws_rows + 31) / 32 * 32;
  int n_split = 0, nsplit = 1;
  int sk_w = 0, sk_grid = 0;
  // (score bias: the split tail on the two-query-tile kernel, no stream-K)
  if (ws != nullptr && !causal && !windowed && (!BIAS || NQ == 2)) {
    if (!BIAS && p.n_tiles < ctas && p.n_tiles <= kMaxSplit) {
      // Stream-K: fewer tiles than CTAs (decode-like shapes).  The key blocks of
      // all tiles are shared out evenly over C CTAs, each with at least
      // kMinPartBlocks of them; C shrinks until the partials fit the workspace.
      const long long W = static_cast<long long>(p.n_tiles) * p.nkb;
      long long C = W / kMinPartBlocks < ctas ? W / kMinPartBlocks : ctas;
      while (C > p.n_tiles &&
             ws_layout(D, p.ws_rows, static_cast<int>(C) + p.n_tiles, 1).total > ws_bytes)
        C -= (C - p.n_tiles + 7) / 8;
      if (C > p.n_tiles && (W + 1) * C < (1ll << 31)) {  // the kernel's index math is 32-bit
        sk_w = static_cast<int>(W);
        sk_grid = static_cast<int>(C);
      }
    } else {
      // Split tail: if the last round of tiles would keep at most half of the
      // CTAs busy, give each of those tiles to two CTAs, one per half of the key
      // blocks.  With coalesced partials and a merge that keeps its loads in
      // flight this pays from 16 key blocks on (the LLaMA-7B layer shape:
      // +5 %); below kMinSplitBlocks the halves are too short for it.
      const int grid0 = p.n_tiles < ctas ? p.n_tiles : ctas;
      const int rem = p.n_tiles % grid0;
      if (p.nkb >= kMinSplitBlocks && p.n_tiles > grid0 && rem > 0 && 2 * rem <= grid0 &&
          rem <= kMaxSplit) {
        n_split = rem;
        nsplit = 2;
      }
    }
  }
  if (n_split > 0 || sk_w > 0) {
    const WsLayout L = sk_w > 0 ? ws_layout(D, p.ws_rows, sk_grid + p.n_tiles, 1)
                                : ws_layout(D, p.ws_rows, n_split, nsplit);
    if (ws_bytes < L.total) {  // split tail only: stream-K was sized to fit
      if (mode == Scratch::kStatic) return FA_ERR_SCRATCH_TOO_SMALL;
      n_split = 0;
      nsplit = 1;
    } else {
      if (mode == Scratch::kStatic &&
          cudaMemsetAsync(ws, 0, L.ml_off, stream) != cudaSuccess)  // the counters start at zero
        return FA_ERR_LAUNCH;
      char* base = static_cast<char*>(ws);
      p.ws_o = reinterpret_cast<float4*>(base + L.o_off);
      p.ws_ml = reinterpret_cast<float4*>(base + L.ml_off);
      p.ws_cnt = reinterpret_cast<int*>(base + L.cnt_off);
    }
  }
  if (n_split == 0 && sk_w == 0) {
    p.ws_o = nullptr;
    p.ws_ml = nullptr;
    p.ws_cnt = nullptr;
  }
  p.sk_w = sk_w;
  p.nsplit = nsplit;
  p.n_whole = sk_w > 0 ? 0 : p.n_tiles - n_split;
  p.n_units = sk_w > 0 ? sk_grid + p.n_tiles : p.n_whole + nsplit * n_split;
  const int grid = sk_w > 0 ? sk_grid : (p.n_units < ctas ? p.n_units : ctas);
  // Dynamic schedule for launches with a workspace in which a CTA gets several
  // units: each CTA takes the next unit of the heavy-first list when it is free
  // (greedy longest-first).  Causal launches use it only up to 8 units per CTA:
  // with few units the static zig-zag leaves CTAs idle at the end (-3 % at
  // N = 4096), with many it balances as well and measured faster.  Stream-K
  // fixes each CTA's units.
  p.sched = nullptr;
  if (ws != nullptr && sk_w == 0 && ws_bytes >= ws_layout(D, 0, 0, 0).ml_off &&
      p.n_units > grid && (!causal || p.n_units <= 8 * grid))
    p.sched = reinterpret_cast<int*>(static_cast<char*>(ws) + kMaxSplit * 2 * 4 * sizeof(int));
  p.use_ring = (p.sched != nullptr || sk_w > 0) ? 1 : 0;
  CUtensorMap tb = tk;  // (unused without a bias)
  int bias_mode = 0;
  if (BIAS) {
    if (!make_bias_map(&tb, *bias, B, Hq, Nq, Nk, BF16)) return FA_ERR_DRIVER;
    bias_mode = (bias->sq ? 0 : fa::kBiasRowBcast) | (bias->sh ? fa::kBiasPerHead : 0) |
                (bias->sb ? fa::kBiasPerBatch : 0);
  }
  fa::fa_fwd_kernel<D, NQ, BF16, BIAS, WIN, STG><<<grid, fa::kThreads, kSmem, stream>>>(
      tq, tq4, tk, tv, p, tb, bias_mode);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

}  // namespace

extern "C" {

const char* fa_status_string(int s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_NULL_POINTER: return "null pointer among q, k, v, o";
    case FA_ERR_MISALIGNED: return "q, k, v, o must be 16-byte aligned and lse 4-byte aligned";
    case FA_ERR_BAD_SHAPE: return "B, Hq, Hkv, Nq, Nk must be >= 1 and sizes must fit";
    case FA_ERR_BAD_GROUPING: return "Hq must be a multiple of Hkv";
    case FA_ERR_UNSUPPORTED_HEAD_DIM: return "head_dim must be 64, 128 or 256";
    case FA_ERR_BAD_SCALE: return "scale must be finite";
    case FA_ERR_BAD_DTYPE: return "dtype must be FA_FP16 or FA_BF16";
    case FA_ERR_NO_DEVICE: return "no current CUDA device of compute capability 10.x (sm_100)";
    case FA_ERR_LAUNCH: return "kernel launch failed";
    case FA_ERR_DRIVER: return "tensor-map encoding failed in the CUDA driver";
    case FA_ERR_DEVICE_TIMEOUT: return "a kernel wait reached its time limit";
    case FA_ERR_OVERLAP: return "o or lse overlaps q, k or v";
    case FA_ERR_SCRATCH_TOO_SMALL:
      return "fa_fwd_noalloc: this problem needs more scratch than the static buffer holds; "
             "use fa_fwd_ws";
    case FA_ERR_BAD_WORKSPACE:
      return "workspace missing, misaligned or smaller than the entry point's *_workspace_size()";
    case FA_ERR_LIBRARY: return "fa_fwd_unfused: a cuBLAS call failed";
    case FA_ERR_BAD_WINDOW:
      return "key window bounds must be >= -1, and a causal launch cannot have window_right > 0";
    default: return "unknown status";
  }
}

long long fa_fwd_num_tiles(int B, int Hq, int Nq, int D) {
  if (B < 1 || Hq < 1 || Nq < 1 || (D != 64 && D != 128 && D != 256)) return 0;
  const long long rows = (long long)nq_for(D) * fa::kBM;
  return (long long)B * Hq * ((Nq + rows - 1) / rows);
}

// Argument checks of every forward entry point: host only, before any CUDA call.
static int check_fwd_args(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                          int Hq, int Hkv, int Nq, int Nk, int D, float scale, int causal,
                          int dtype, int wl, int wr) {
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_BAD_DTYPE;
  if (wl < -1 || wr < -1 || (causal && wr > 0)) return FA_ERR_BAD_WINDOW;
  if (D != 64 && D != 128 && D != 256) return FA_ERR_UNSUPPORTED_HEAD_DIM;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1) return FA_ERR_BAD_SHAPE;
  if (Hq % Hkv != 0) return FA_ERR_BAD_GROUPING;
  const long long qo_elems = (long long)B * Hq * Nq * D, kv_elems = (long long)B * Hkv * Nk * D;
  // work-tile count, row indices and TMA coordinates are 32-bit
  if ((long long)B * Hq * Nq >= (1ll << 31) || (long long)B * Hkv * Nk >= (1ll << 31))
    return FA_ERR_BAD_SHAPE;
  if (!std::isfinite(scale)) return FA_ERR_BAD_SCALE;
  if (!q || !k || !v || !o) return FA_ERR_NULL_POINTER;
  if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)o) & 15u) return FA_ERR_MISALIGNED;
  if (lse && ((uintptr_t)lse & 3u)) return FA_ERR_MISALIGNED;
  const size_t qo_b = (size_t)qo_elems * 2, kv_b = (size_t)kv_elems * 2;
  if (overlaps(o, qo_b, q, qo_b) || overlaps(o, qo_b, k, kv_b) || overlaps(o, qo_b, v, kv_b))
    return FA_ERR_OVERLAP;
  if (lse) {
    const size_t lb = (size_t)B * Hq * Nq * 4;
    if (overlaps(lse, lb, q, qo_b) || overlaps(lse, lb, k, kv_b) || overlaps(lse, lb, v, kv_b) ||
        overlaps(lse, lb, o, qo_b))
      return FA_ERR_OVERLAP;
  }
  return FA_OK;
}

static int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                    int Hkv, int Nq, int Nk, int D, float scale, int causal, void* stream, int dtype,
                    void* ws, size_t ws_bytes, Scratch mode = Scratch::kCaller, int wl = -1,
                    int wr = -1, const BiasArg* bias = nullptr) {
  const int bad = check_fwd_args(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal, dtype, wl, wr);
  if (bad != FA_OK) return bad;
  // ---- device
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_NO_DEVICE;
  DeviceState& ds = g_dev[dev];
  std::call_once(ds.once, [&] {
    int major = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    ds.sm100 = (major == 10);
    ds.sms = sms;
  });
  if (!ds.sm100 || ds.sms < 1) return FA_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = dtype == FA_BF16;
  // A work tile of at most 128 rows (short queries, or a packed GQA group) runs
  // the one-query-tile kernel: its two S buffers let the softmax of key block j
  // overlap the S MMA of block j + 1, and its K/V staging is deeper.
  if (bias != nullptr) {  // score bias: the kernels with bias staging
#define FA_BARGS q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal, wl, wr, st, dev, ws, ws_bytes, \
                 Scratch::kCaller, bias
    // more than 128 query rows (D <= 128) and no key window: the two-query-tile
    // kernel; key windows: the one-query-tile kernels, which take them per tile
    const bool win = wl >= 0 || wr >= 0;
    if (D == 64 && Nq > fa::kBM && !win)
      return bf ? launch<64, 2, true, true>(FA_BARGS) : launch<64, 2, false, true>(FA_BARGS);
    if (D == 128 && Nq > fa::kBM && !win)
      return bf ? launch<128, 2, true, true>(FA_BARGS) : launch<128, 2, false, true>(FA_BARGS);
    switch (D) {
      case 64: return bf ? launch<64, 1, true, true>(FA_BARGS) : launch<64, 1, false, true>(FA_BARGS);
      case 128: return bf ? launch<128, 1, true, true>(FA_BARGS) : launch<128, 1, false, true>(FA_BARGS);
      default: return bf ? launch<256, 1, true, true>(FA_BARGS) : launch<256, 1, false, true>(FA_BARGS);
    }
#undef FA_BARGS
  }
  // Windowed launches: each query tile gets its own key block range; tiles of
  // 256 rows (D <= 128) run the two-query-tile kernel's windowed variant.
  const bool windowed = wl >= 0 || wr >= 0;
  if (windowed && D <= 128 && Nq > fa::kBM) {
#define FA_WARGS q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal, wl, wr, st, dev, ws, ws_bytes, mode
    if (D == 64)
      return bf ? launch<64, 2, true, false, true>(FA_WARGS) : launch<64, 2, false, false, true>(FA_WARGS);
    return bf ? launch<128, 2, true, false, true>(FA_WARGS) : launch<128, 2, false, false, true>(FA_WARGS);
#undef FA_WARGS
  }
  // ... and so does a problem too small to give half of the CTAs a 256-row
  // tile: 128-row tiles double the CTAs that take part (short sequences).
  const long long tiles2 = (long long)B * Hq * ((Nq + 2 * fa::kBM - 1) / (2 * fa::kBM));
  const int cap = g_max_ctas.load();
  const int ctas = (cap > 0 && cap < ds.sms) ? cap : ds.sms;
  const bool one_tile = windowed ||
                        (pack_heads(Hq, Hkv, Nq, causal) ? (Hq / Hkv) * Nq : Nq) <= fa::kBM ||
                        2 * tiles2 < ctas;
#define FA_ARGS q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal, wl, wr, st, dev, ws, ws_bytes, mode
  switch (D) {
    case 64:
      if (one_tile) return bf ? launch<64, 1, true>(FA_ARGS) : launch<64, 1, false>(FA_ARGS);
      return bf ? launch<64, 2, true>(FA_ARGS) : launch<64, 2, false>(FA_ARGS);
    case 128:
      if (one_tile) return bf ? launch<128, 1, true>(FA_ARGS) : launch<128, 1, false>(FA_ARGS);
      // fp16 without a mask, rows of at most kStagedMaxKeys keys: the staged
      // epilogue (output written as whole lines; the epilogue is a larger share
      // of such a short tile)
      if (!bf && !causal && Nk <= kStagedMaxKeys) return launch<128, 2, false, false, false, true>(FA_ARGS);
      return bf ? launch<128, 2, true>(FA_ARGS) : launch<128, 2, false>(FA_ARGS);
    default:
      return bf ? launch<256, 1, true>(FA_ARGS) : launch<256, 1, false>(FA_ARGS);
  }
#undef FA_ARGS
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
           int Hkv, int Nq, int Nk, int D, float scale, int causal, void* stream, int dtype) {
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal, stream, dtype, nullptr, 0);
}

int fa_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                  int Hkv, int Nq, int Nk, int D, float scale, int causal, int window_left,
                  int window_right, void* stream, int dtype, void* workspace,
                  size_t workspace_bytes) {
  if (workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return FA_ERR_MISALIGNED;
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal, stream, dtype,
                  workspace, workspace != nullptr ? workspace_bytes : 0, Scratch::kCaller,
                  window_left, window_right);
}

int fa_fwd_bias_ws(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                   int Hkv, int Nq, int Nk, int D, float scale, int causal, const void* bias,
                   long long bias_stride_b, long long bias_stride_h, long long bias_stride_q,
                   int window_left, int window_right, void* stream, int dtype, void* workspace,
                   size_t workspace_bytes) {
  if (bias == nullptr) return FA_ERR_NULL_POINTER;
  if (workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return FA_ERR_MISALIGNED;
  if (bias_stride_b < 0 || bias_stride_h < 0 || bias_stride_q < 0) return FA_ERR_BAD_SHAPE;
  if ((reinterpret_cast<uintptr_t>(bias) & 15u) || (bias_stride_b & 7) || (bias_stride_h & 7) ||
      (bias_stride_q & 7))
    return FA_ERR_MISALIGNED;
  if (B >= 1 && Hq >= 1 && Nq >= 1 && Nk >= 1 && o != nullptr) {  // o, lse must not overlap the bias
    const size_t extent = 2 * static_cast<size_t>((B - 1) * bias_stride_b + (Hq - 1) * bias_stride_h +
                                                  (Nq - 1) * bias_stride_q + Nk);
    if (overlaps(o, (size_t)B * Hq * Nq * D * 2, bias, extent) ||
        (lse && overlaps(lse, (size_t)B * Hq * Nq * 4, bias, extent)))
      return FA_ERR_OVERLAP;
  }
  if (workspace != nullptr && B >= 1 && Hq >= 1 && Nq >= 1 && Nk >= 1) {  // nor the workspace
    const size_t extent = 2 * static_cast<size_t>((B - 1) * bias_stride_b + (Hq - 1) * bias_stride_h +
                                                  (Nq - 1) * bias_stride_q + Nk);
    if (overlaps(workspace, workspace_bytes, bias, extent)) return FA_ERR_OVERLAP;
  }
  const BiasArg a{bias, bias_stride_b, bias_stride_h, bias_stride_q};
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal, stream, dtype, workspace,
                  workspace != nullptr ? workspace_bytes : 0, Scratch::kCaller, window_left,
                  window_right, &a);
}

int fa_fwd_bias_window(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int Hq, int Hkv, int Nq, int Nk, int D, float scale, int causal,
                       const void* bias, long long bias_stride_b, long long bias_stride_h,
                       long long bias_stride_q, int window_left, int window_right, void* stream,
                       int dtype) {
  return fa_fwd_bias_ws(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal, bias, bias_stride_b,
                        bias_stride_h, bias_stride_q, window_left, window_right, stream, dtype,
                        nullptr, 0);
}

int fa_fwd_bias(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                int Hkv, int Nq, int Nk, int D, float scale, int causal, const void* bias,
                long long bias_stride_b, long long bias_stride_h, long long bias_stride_q,
                void* stream, int dtype) {
  return fa_fwd_bias_window(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal, bias,
                            bias_stride_b, bias_stride_h, bias_stride_q, -1, -1, stream, dtype);
}

size_t fa_fwd_workspace_size(int D) {
  if (D != 64 && D != 128 && D != 256) return 0;
  int dev = -1, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 2)
    return 0;
  return ws_layout(D, nq_for(D) * 128, sms / 2 < kMaxSplit ? sms / 2 : kMaxSplit, 2).total;
}

int fa_fwd_ws(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
              int Hkv, int Nq, int Nk, int D, float scale, int causal, void* stream, int dtype,
              void* workspace, size_t workspace_bytes) {
  if (workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return FA_ERR_MISALIGNED;
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal, stream, dtype, workspace,
                  workspace_bytes);
}

// ---- fa_fwd_noalloc: the split-tail launch with library-owned scratch ----------
// For callers that cannot allocate device memory (see include/fa.h): the
// scratch of the split tail lives in this file-scope device array, which every
// GPU that loads the library holds until the process exits.  In host code the
// array's name is only a host-side stand-in, so its device address is fetched
// with cudaGetSymbolAddress, with the device current, by the first call on each
// device (and kept once that lookup has succeeded).
constexpr size_t kNoAllocScratchBytes = size_t(24) << 20;  // 24 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array, per device; kept only once a lookup succeeded,
// so a lookup that failed (for example inside a stream capture) is retried on
// the next call.
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

int fa_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                   int Hkv, int Nq, int Nk, int D, float scale, int causal, void* stream,
                   int dtype) {
  const int bad = check_fwd_args(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal, dtype, -1, -1);
  if (bad != FA_OK) return bad;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_NO_DEVICE;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
        cudaGetLastError();  // the failed lookup leaves no sticky error behind
        return FA_ERR_LAUNCH;
      }
      g_noalloc_ptr[dev] = ptr;
    }
    scratch = g_noalloc_ptr[dev];
  }
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal, stream, dtype, scratch,
                  kNoAllocScratchBytes, Scratch::kStatic);
}

size_t fa_fwd_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

int fa_set_max_ctas(int n) {
  if (n < 0) return FA_ERR_BAD_SHAPE;
  return g_max_ctas.exchange(n);
}

int fa_fwd_fp16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                int Hkv, int Nq, int Nk, int D, float scale, int causal, void* stream) {
  return fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal, stream, FA_FP16);
}

int fa_fwd_bf16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                int Hkv, int Nq, int Nk, int D, float scale, int causal, void* stream) {
  return fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal, stream, FA_BF16);
}

int fa_bwd_device_status_internal(int reset);  // fa_bwd_sm100.cu

int fa_device_status(int reset) {
  unsigned int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(&v, fa::g_status, sizeof(v)) != cudaSuccess) return -1;
  const int vb = fa_bwd_device_status_internal(reset);  // the backward kernels' word
  if (vb < 0) return -1;
  if (reset) {
    const unsigned int z = 0;
    const unsigned long long zz = 0;
    if (cudaMemcpyToSymbol(fa::g_status, &z, sizeof(z)) != cudaSuccess ||
        cudaMemcpyToSymbol(fa::g_timeout_site, &zz, sizeof(zz)) != cudaSuccess)
      return -1;
  }
  return v != 0 ? static_cast<int>(v) : vb;
}

int fa_debug_wait_timeout(void* stream) {
  fa::wait_timeout_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

int fa_debug_exp2_fma(const float* x, float* y, int n, void* stream) {
  if (!x || !y) return FA_ERR_NULL_POINTER;
  if (n < 1) return FA_ERR_BAD_SHAPE;
  const int threads = 256, pairs = (n + 1) / 2;
  fa::exp2_fma_eval_kernel<<<(pairs + threads - 1) / threads, threads, 0,
                             reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

int fa_device_timeout_site(unsigned long long* site) {
  if (!site) return FA_ERR_NULL_POINTER;
  if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_NO_DEVICE;
  if (cudaMemcpyFromSymbol(site, fa::g_timeout_site, sizeof(*site)) != cudaSuccess)
    return FA_ERR_NO_DEVICE;
  return FA_OK;
}

}  // extern "C"
