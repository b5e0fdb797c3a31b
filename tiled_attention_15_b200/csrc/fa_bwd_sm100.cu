// fa_bwd_sm100.cu -- backward pass of the fused attention for B200 (sm_100a).
//
// The pages only say that training has to keep gradients (hwcomputing.csdn.net
// page, section "标准Attention：一次摊开整本词典"); the operation here is the
// exact gradient of the forward pass O = softmax(scale * Q K^T) V for an
// upstream gradient dO, computed the way the forward pass is: tile by tile,
// without materialising the score matrix.  The softmax is recomputed from Q, K
// and the forward pass's row log-sum-exp (LSE):
//
//   P_ij  = exp(scale q_i.k_j - LSE_i)            Delta_i = dO_i . O_i
//   dP_ij = dO_i . v_j                            dS_ij   = P_ij (dP_ij - Delta_i)
//   dV_j  = sum_i P_ij dO_i     dK_j = scale sum_i dS_ij q_i     dQ_i = scale sum_j dS_ij k_j
//
// Three kernels, all with tcgen05 tensor-core MMAs accumulating in tensor
// memory (TMEM) and TMA loads with 128-byte swizzle:
//   * bwd_prep_kernel: Delta = rowsum(dO * O) and LSE * log2(e), into two planes
//     padded to whole 128-row blocks (+inf / 0 in the padding, which zeroes P
//     there without a mask);
//   * bwd_dkdv_kernel: per 128-key tile, a loop over the query blocks of
//     every query head of its GQA group: S^T = K Q^T, dP^T = V dO^T,
//     P^T and dS^T (16-bit, written back over S^T and dP^T), dV += P^T dO,
//     dK += dS^T Q;
//   * bwd_dq_kernel: per 128-query tile, a loop over the key blocks:
//     S = Q K^T, dP = dO V^T, dS, dQ += dS K.
// Both are persistent (one CTA per SM, tiles in a snake order): a tile's
// loads and first MMAs overlap the previous tile's epilogue.
// dQ is computed in its own pass (S and dP recomputed: two extra MMAs per block
// pair) instead of being accumulated across key tiles with atomics: no atomic
// traffic, and the result does not depend on the order CTAs finish in.
// Head dimension 256 has its own three kernels (end of the device code): the
// streamed operand in 64-row blocks, and dV and dK from separate launches.
//
// Warp roles (384 threads, one CTA per SM): warps 0-7 two compute warpgroups
// that split each block's 128 columns into halves (warp w reads TMEM lanes
// 32 (w % 4) .. +31), warp 8 issues the MMAs (one thread), warp 9 issues the
// TMA loads (one thread), warps 10-11 idle.  Every mbarrier wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>
#include <utility>

#include "fa.h"
#include "sm100_ptx.cuh"

namespace fab {
using namespace fa;

constexpr int kBM = 128;  // query rows per block
constexpr int kBN = 128;  // keys per block
constexpr int kThreads = 384;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait
constexpr float kLog2e = 1.4426950408889634f;
// score bias broadcast (bias_mode bits): one row for every query; per query
// head; per batch entry (a dimension without its bit has stride 0)
constexpr int kBiasRowBcast = 1, kBiasPerHead = 2, kBiasPerBatch = 4;
constexpr int kBiasTileBytes = 128 * 128 * 2;  // [2 boxes][128 rows][64 keys], 16-bit

// Programmatic dependent launch: let the next kernel in the stream (launched
// with programmatic stream serialisation) start; wait until the kernels this
// one depends on have completed and their writes are visible.
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ unsigned int g_bwd_status = 0;
__device__ unsigned long long g_bwd_site = 0;

// 1-D bulk copy global -> shared, completion counted on `bar` in bytes (both
// addresses 16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity,
                                         volatile uint32_t* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      const uint32_t site =
          0x80000000u | ((threadIdx.x >> 5) << 24) | ((bar & 0x3FFFFu) << 1) | parity;
      atomicCAS(const_cast<uint32_t*>(abort_flag), 0u, site);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void publish_abort(uint32_t flag) {
  if (flag == 0u) return;
  if (atomicCAS(&g_bwd_status, 0u, static_cast<unsigned>(FA_ERR_DEVICE_TIMEOUT)) == 0u)
    g_bwd_site = (static_cast<unsigned long long>(blockIdx.x) << 48) |
                 (static_cast<unsigned long long>((flag >> 24) & 0x3Fu) << 40) |
                 (static_cast<unsigned long long>((flag >> 1) & 0x3FFFFu) << 8) | (flag & 1u);
}

__device__ __forceinline__ uint32_t pack2(float a, float b, bool bf16) {
  if (bf16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// one 16-bit value (fp16 or bf16) from shared memory, as float
__device__ __forceinline__ float bias_at(uint32_t saddr, bool bf16) {
  unsigned short h;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h) : "r"(saddr));
  return bf16 ? __uint_as_float(static_cast<uint32_t>(h) << 16) : __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ float2 unpack2(uint32_t w, bool bf16) {
  if (bf16) return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w));
  return __half22float2(*reinterpret_cast<__half2*>(&w));
}

struct BwdParams {
  void* dq;
  void* dk;
  void* dv;
  const float* lse2;   // [B*Hq][Nq_pad] LSE * log2(e); +inf in the padding
  const float* delta;  // [B*Hq][Nq_pad] rowsum(dO * O); 0 in the padding
  int B, Hq, Hkv, Nq, Nk, Nq_pad, group, causal;
  // key window: query i sees keys i - wl .. i + wr (-1: no bound); wr is 0 when causal
  int wl, wr;
  float c;      // scale * log2(e)
  float scale;
  int nqt, nkt;  // query / key blocks per head
};

// ------------------------------------------------------------------ Delta, LSE2
// D / 8 threads per row, 8 elements (16 bytes) each; rows in the padding get
// (+inf, 0).  Rows are taken warp by warp so that every lane of a warp reaches
// the shuffles, kPrepGroups row groups per pass with all their loads issued
// before any is used (more bytes in flight per thread).
constexpr int kPrepGroups = 4;
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const uint16_t* __restrict__ o,
                                                       const uint16_t* __restrict__ dout,
                                                       const float* __restrict__ lse,
                                                       float* __restrict__ lse2,
                                                       float* __restrict__ delta, int BH, int Nq,
                                                       int Nq_pad) {
  constexpr int TPR = D / 8;      // threads per row
  constexpr int RPW = 32 / TPR;   // rows per warp and group
  constexpr int U = kPrepGroups;
  grid_dep_launch();  // the dK/dV kernel may start its setup and K/V loads
  const long long total = static_cast<long long>(BH) * Nq_pad;
  const int lane = threadIdx.x & 31, sub = lane % TPR;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long base = warp * RPW * U; base < total; base += n_warps * RPW * U) {
    uint4 a[U], b[U];
    float L[U];
    bool live[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long row = base + u * RPW + lane / TPR;
      const long long bh = row / Nq_pad;
      const int i = static_cast<int>(row - bh * Nq_pad);
      live[u] = row < total && i < Nq;
      a[u] = b[u] = make_uint4(0u, 0u, 0u, 0u);
      L[u] = -INFINITY;
      if (live[u]) {
        const size_t off = (static_cast<size_t>(bh) * Nq + i) * D + sub * 8;
        a[u] = __ldg(reinterpret_cast<const uint4*>(o + off));
        b[u] = __ldg(reinterpret_cast<const uint4*>(dout + off));
        L[u] = __ldg(lse + bh * Nq + i);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long row = base + u * RPW + lane / TPR;
      float acc = 0.f;
      if (live[u]) {
        const uint32_t aw[4] = {a[u].x, a[u].y, a[u].z, a[u].w}, bw[4] = {b[u].x, b[u].y, b[u].z, b[u].w};
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float2 fa2 = unpack2(aw[x], BF16), fb2 = unpack2(bw[x], BF16);
          acc = fmaf(fa2.x, fb2.x, acc);
          acc = fmaf(fa2.y, fb2.y, acc);
        }
      }
#pragma unroll
      for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (sub == 0 && row < total) {
        delta[row] = live[u] ? acc : 0.f;
        // a row that saw no key (LSE = -inf, key windows) gets +inf: P = 0 there
        lse2[row] = L[u] == -INFINITY ? INFINITY : L[u] * kLog2e;
      }
    }
  }
}

// ------------------------------------------------------------------ shared pieces
struct Ctx {
  uint32_t sbase;
  uint32_t tmem;
  volatile uint32_t* abort_flag;
  __device__ uint32_t bar(int i, int off_bar) const { return sbase + off_bar + 8u * i; }
};

// S-type MMA over one 128 x D by 128 x D pair of K-major SW128 tiles:
// D[128 x 128] = A B^T.
template <int D>
__device__ __forceinline__ void mma_nt(uint32_t d, uint64_t a0, uint64_t b0, uint32_t idesc,
                                       int chunk_a, int chunk_b) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off_a = ((kk >> 2) * chunk_a + (kk & 3) * 32) >> 4;
    const uint32_t off_b = ((kk >> 2) * chunk_b + (kk & 3) * 32) >> 4;
    mma_ss(d, a0 + off_a, b0 + off_b, idesc, kk > 0 ? 1u : 0u);
  }
}

// Accumulating MMA with A (16-bit, 128 rows x 128 columns of K) in tensor
// memory and B an MN-major SW128 tile (128 rows of K, D columns).  The packed A
// of K index k sits at column acol(k / 16) + (k % 16) / 2.
template <int D, typename ACol>
__device__ __forceinline__ void mma_tn(uint32_t d, uint32_t a, uint64_t b0, uint32_t idesc,
                                       bool acc, ACol acol) {
#pragma unroll
  for (int kk = 0; kk < 128 / 16; ++kk)
    mma_ts(d, a + acol(kk), b0 + static_cast<uint64_t>((kk * 2048) >> 4), idesc,
           (acc || kk > 0) ? 1u : 0u);
}

// ================================================================== dK, dV
template <int D, bool BIAS = false>
struct GeoKV {
  static constexpr int DCH = D / 64;
  static constexpr int T_BYTES = 128 * D * 2;  // one 128-row tile
  static constexpr int CHUNK = 128 * 128;      // one 64-column chunk of a tile
  // Q and dO tiles stream through a ring of single-tile slots in the order
  // Q0 dO0 Q1 dO1 ...; a slot holding Q_n also holds that block's lse2 and
  // delta (1 KB side buffer).  dO_n is freed after dV(n), Q_n after dK(n).
  // (a score bias takes one slot's room at head_dim 128 for its tile)
  static constexpr int NSLOT = D == 64 ? 8 : (BIAS ? 3 : 4);
  static constexpr int SLOT_BYTES = T_BYTES + 1024;
  static constexpr int OFF_K = 0, OFF_V = T_BYTES, OFF_SL = 2 * T_BYTES;
  static constexpr int OFF_BIAS = OFF_SL + NSLOT * SLOT_BYTES;  // the block pair's bias tile
  static constexpr int OFF_BAR = OFF_BIAS + (BIAS ? kBiasTileBytes : 0);
  // barriers (the kernel is persistent: B_KVE = the tile's K and V no longer
  // read, B_ACCE = its dV and dK read out of tensor memory, B_STG = its
  // epilogue done with the staging slots)
  static constexpr int B_KV = 0, B_SLF = 1, B_SLE = 1 + NSLOT, B_SF = 1 + 2 * NSLOT,
                       B_DPF = B_SF + 1, B_PF = B_SF + 2, B_DSF = B_SF + 3, B_ACC = B_SF + 4,
                       B_BF = B_SF + 5, B_BE = B_SF + 6, B_KVE = B_SF + 7, B_ACCE = B_SF + 8,
                       B_STG = B_SF + 9, NBAR = B_SF + 10;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  // TMEM columns: S^T 0..127 (P^T over it), dP^T 128..255 (dS^T over it), dV, dK
  static constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + D;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(256 + 2 * D <= 512, "tensor memory budget");
};

struct KVTile {
  int bkv;  // b * Hkv + kv head
  int kt;   // key block
  int i0;   // first query block
  int nqb;  // query blocks per head
  int nb;   // blocks: group heads x query blocks
};

// The tile a persistent CTA takes in round r (snake order over the grid).
__device__ __forceinline__ int snake_tile(int r) {
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  return r * G + ((r & 1) ? G - 1 - c : c);
}

// tile t; bq: rows of a query block (128, or 64 at head_dim 256)
__device__ __forceinline__ KVTile kv_tile(const BwdParams& p, int t, int bq = kBM) {
  KVTile T;
  const int BK = p.B * p.Hkv;
  if (p.causal) {  // small key blocks see the most query blocks: run them first
    T.kt = t / BK;
    T.bkv = t % BK;
  } else {
    T.bkv = t / p.nkt;
    T.kt = t % p.nkt;
  }
  // query blocks that see a key of this tile: q >= k0 - wr and q <= k0 + 127 + wl
  // (causal: wr = 0, so from the diagonal block on; top-left aligned)
  const int k0 = T.kt * kBN, nqblk = p.Nq_pad / bq;
  T.i0 = p.wr >= 0 ? max(0, k0 - p.wr) / bq : 0;
  const int i1 = p.wl >= 0 ? min(nqblk - 1, (k0 + kBN - 1 + p.wl) / bq) : nqblk - 1;
  T.nqb = i1 >= T.i0 ? i1 - T.i0 + 1 : 0;
  T.nb = p.group * T.nqb;
  return T;
}

// Persistent: in round r CTA c takes tile r G + c (r even) or r G + G - 1 - c
// (r odd), G = gridDim.x -- the tiles come heaviest first (causal), so the
// snake order evens out each CTA's sum.  Ring items, block
// indices and tile indices run on across tiles (the barrier phases follow
// them), so the next tile's K, V and first Q / dO blocks load, and its first
// S^T and dP^T run, while the compute warps write the previous tile's dK, dV.
// The epilogue stages its rows in the two slots the next tile's ring items
// reach last (items M + NSLOT - 2 and M + NSLOT - 1, M = the first item after
// the tile): they held the tile's own last Q and dO, so they are idle once its
// accumulators are final, and the TMA thread loads into them only after
// B_STG.  Tiles no query sees (key windows) write zeros and take no part in
// the barriers.
template <int D, bool BF16, bool BIAS = false>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const BwdParams p, const __grid_constant__ CUtensorMap tm_b, const int bias_mode) {
  using G = GeoKV<D, BIAS>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  uint32_t* misc = reinterpret_cast<uint32_t*>(gbase + G::OFF_MISC);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Ctx cx;
  cx.sbase = sbase;
  cx.abort_flag = misc + 1;
  auto B = [&](int i) { return cx.bar(i, G::OFF_BAR); };
  const int n_tiles = p.B * p.Hkv * p.nkt;

  if (threadIdx.x == 0) {
    mbar_init(B(G::B_KV), 1);
    for (int s = 0; s < G::NSLOT; ++s) {
      mbar_init(B(G::B_SLF + s), 1);
      mbar_init(B(G::B_SLE + s), 1);
    }
    mbar_init(B(G::B_SF), 1);
    mbar_init(B(G::B_DPF), 1);
    mbar_init(B(G::B_PF), 8);
    mbar_init(B(G::B_DSF), 8);
    mbar_init(B(G::B_ACC), 1);
    mbar_init(B(G::B_BF), 1);
    mbar_init(B(G::B_BE), 8);
    mbar_init(B(G::B_KVE), 1);
    mbar_init(B(G::B_ACCE), 8);
    mbar_init(B(G::B_STG), 8);
    misc[1] = 0u;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(misc), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cx.tmem = misc[0];

  // every CTA is resident: the dQ kernel may launch (it waits for this one
  // before it reads anything this call writes)
  if (threadIdx.x == 0) grid_dep_launch();
  // Registers: 208 for the two compute warpgroups, 88 for the rest (2 x 128 x
  // 208 + 128 x 88 = 384 x 168); each role branch sets its own limit.
  if (warp >= 8) setmaxnreg_dec<88>();
  if (warp == 9 && lane == 0) {
    // ---- TMA: per tile K and V, then (Q, dO, lse2, delta) per query block.
    // lse2 and delta come from the prep kernel, which may still be running
    // (programmatic launch): its writes are waited for before the first of them.
    bool dep = false;
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_do);
    const uint64_t pol_first = policy_evict_first(), pol_last = policy_evict_last();
    uint32_t m0 = 0;                    // ring items issued before this tile
    uint32_t gate = 0xffffffffu;        // first item that must wait for an epilogue's staging
    uint32_t gate_par = 0;              // ... and that epilogue's B_STG phase
    int it = 0;                         // tiles with blocks before this one
    bool ok = true;
    for (int rd = 0; ok && rd * static_cast<int>(gridDim.x) < n_tiles; ++rd) {
      const int t = snake_tile(rd);
      if (t >= n_tiles) continue;
      const KVTile T = kv_tile(p, t);
      if (T.nb == 0) continue;
      if (it > 0 && !wait_bar(B(G::B_KVE), (it - 1) & 1u, cx.abort_flag)) break;
      const int kv_row0 = T.kt * kBN;
      mbar_arrive_expect_tx(B(G::B_KV), 2 * G::T_BYTES);
#pragma unroll
      for (int c = 0; c < G::DCH; ++c) {
        tma_load_3d(sbase + G::OFF_K + c * G::CHUNK, &tm_k, B(G::B_KV), c * 64, kv_row0, T.bkv, pol_first);
        tma_load_3d(sbase + G::OFF_V + c * G::CHUNK, &tm_v, B(G::B_KV), c * 64, kv_row0, T.bkv, pol_first);
      }
      if (!dep) {
        grid_dep_wait();
        dep = true;
      }
      const int nqb = T.nqb;
      for (int mm = 0; mm < 2 * T.nb; ++mm) {  // item mm: Q (even, + lse2, delta) or dO (odd) of block mm / 2
        const uint32_t m = m0 + static_cast<uint32_t>(mm);
        if (m == gate && !wait_bar(B(G::B_STG), gate_par, cx.abort_flag)) { ok = false; break; }
        const int sl = static_cast<int>(m % G::NSLOT), n = mm >> 1;
        if (m >= (uint32_t)G::NSLOT &&
            !wait_bar(B(G::B_SLE + sl), ((m / G::NSLOT) - 1) & 1u, cx.abort_flag)) { ok = false; break; }
        const int h = n / nqb, i = T.i0 + n % nqb;
        const int bh = (T.bkv / p.Hkv) * p.Hq + (T.bkv % p.Hkv) * p.group + h;
        const uint32_t sb = sbase + G::OFF_SL + sl * G::SLOT_BYTES;
        mbar_arrive_expect_tx(B(G::B_SLF + sl), G::T_BYTES + ((mm & 1) ? 0 : 1024));
#pragma unroll
        for (int c = 0; c < G::DCH; ++c)
          tma_load_3d(sb + c * G::CHUNK, (mm & 1) ? &tm_do : &tm_q, B(G::B_SLF + sl), c * 64, i * kBM,
                      bh, pol_last);
        if ((mm & 1) == 0) {
          const size_t row = static_cast<size_t>(bh) * p.Nq_pad + static_cast<size_t>(i) * kBM;
          bulk_load(sb + G::T_BYTES, p.lse2 + row, 512, B(G::B_SLF + sl));
          bulk_load(sb + G::T_BYTES + 512, p.delta + row, 512, B(G::B_SLF + sl));
        }
      }
      if (!ok) break;
      m0 += 2u * static_cast<uint32_t>(T.nb);
      // a previous epilogue's gate not reached by this tile's items (short
      // tiles): wait for it here, before this tile's gate replaces it
      if (gate != 0xffffffffu && gate >= m0 && !wait_bar(B(G::B_STG), gate_par, cx.abort_flag)) break;
      gate = m0 + G::NSLOT - 2;
      gate_par = static_cast<uint32_t>(it) & 1u;
      ++it;
    }
    if (!dep) grid_dep_wait();  // (no tile with blocks: still no earlier exit than prep)
  } else if (BIAS && warp == 10 && lane == 0) {
    // ---- TMA: the bias tile of each (query block, key tile) pair: rows = the
    // block's queries (one row if broadcast over queries), columns = the tile's keys
    const uint64_t pol = policy_evict_last();
    const int rows = (bias_mode & kBiasRowBcast) ? 1 : kBM;
    uint32_t g0 = 0;  // blocks before this tile
    bool ok = true;
    for (int rd = 0; ok && rd * static_cast<int>(gridDim.x) < n_tiles; ++rd) {
      const int t = snake_tile(rd);
      if (t >= n_tiles) continue;
      const KVTile T = kv_tile(p, t);
      if (T.nb == 0) continue;
      const int b = T.bkv / p.Hkv, kv_row0 = T.kt * kBN;
      for (int n = 0; n < T.nb; ++n) {
        const uint32_t g = g0 + static_cast<uint32_t>(n);
        if (g > 0 && !wait_bar(B(G::B_BE), (g - 1) & 1u, cx.abort_flag)) { ok = false; break; }
        const int hq = (T.bkv % p.Hkv) * p.group + n / T.nqb, i = T.i0 + n % T.nqb;
        mbar_arrive_expect_tx(B(G::B_BF), 2 * rows * 128);
#pragma unroll
        for (int box = 0; box < 2; ++box)
          tma_load_4d(sbase + G::OFF_BIAS + box * (kBiasTileBytes / 2), &tm_b, B(G::B_BF),
                      kv_row0 + box * 64, (bias_mode & kBiasRowBcast) ? 0 : i * kBM,
                      (bias_mode & kBiasPerHead) ? hq : 0, (bias_mode & kBiasPerBatch) ? b : 0, pol);
      }
      g0 += static_cast<uint32_t>(T.nb);
    }
  } else if (warp == 8 && lane == 0) {
    // ---- MMA, per tile: S(0) dP(0) | dV(n) S(n+1) dK(n) dP(n+1) | ...
    constexpr uint32_t kIdNT = idesc_f16(128, 128, BF16, false);
    constexpr uint32_t kIdTN = idesc_f16(128, D, BF16, true);
    const uint32_t tm = cx.tmem;
    const uint64_t dk0 = sdesc_sw128(sbase + G::OFF_K, 16, 1024);
    const uint64_t dv0 = sdesc_sw128(sbase + G::OFF_V, 16, 1024);
    auto st_desc = [&](uint32_t m, bool mn) {  // ring item m: a Q (even) or dO (odd) block
      const uint32_t a = sbase + G::OFF_SL + (m % G::NSLOT) * G::SLOT_BYTES;
      return mn ? sdesc_sw128(a, G::CHUNK, 1024) : sdesc_sw128(a, 16, 1024);
    };
    auto wait_item = [&](uint32_t m) {
      return wait_bar(B(G::B_SLF + m % G::NSLOT), (m / G::NSLOT) & 1u, cx.abort_flag);
    };
    // P^T / dS^T of query column q: warpgroup q / 64 packed its half at its own
    // first 32 columns -> K step kk (16 queries) at (kk / 4) * 64 + (kk % 4) * 8
    auto acol = [](int kk) { return static_cast<uint32_t>((kk >> 2) * 64 + (kk & 3) * 8); };
    uint32_t m0 = 0, g0 = 0;
    int it = 0;
    bool ok = true;
    for (int rd = 0; ok && rd * static_cast<int>(gridDim.x) < n_tiles; ++rd) {
      const int t = snake_tile(rd);
      if (t >= n_tiles) continue;
      const KVTile T = kv_tile(p, t);
      if (T.nb == 0) continue;
      ok = wait_bar(B(G::B_KV), static_cast<uint32_t>(it) & 1u, cx.abort_flag) && wait_item(m0) &&
           wait_item(m0 + 1);
      if (!ok) break;
      tc_fence_after();
      mma_nt<D>(tm + G::T_S, dk0, st_desc(m0, false), kIdNT, G::CHUNK, G::CHUNK);
      mma_commit(B(G::B_SF));
      mma_nt<D>(tm + G::T_DP, dv0, st_desc(m0 + 1, false), kIdNT, G::CHUNK, G::CHUNK);
      mma_commit(B(G::B_DPF));
      if (T.nb == 1) mma_commit(B(G::B_KVE));
      for (int n = 0; n < T.nb; ++n) {
        const uint32_t g = g0 + static_cast<uint32_t>(n), m = m0 + 2u * static_cast<uint32_t>(n);
        if (!wait_bar(B(G::B_PF), g & 1u, cx.abort_flag)) { ok = false; break; }
        // the first dV of a tile overwrites the accumulators: the previous
        // tile's epilogue must have read them out
        if (n == 0 && it > 0 && !wait_bar(B(G::B_ACCE), (it - 1) & 1u, cx.abort_flag)) { ok = false; break; }
        tc_fence_after();
        mma_tn<D>(tm + G::T_DV, tm + G::T_S, st_desc(m + 1, true), kIdTN, n > 0, acol);
        mma_commit(B(G::B_SLE + (m + 1) % G::NSLOT));  // dO_n's slot
        if (n + 1 < T.nb) {
          if (!wait_item(m + 2)) { ok = false; break; }
          tc_fence_after();
          mma_nt<D>(tm + G::T_S, dk0, st_desc(m + 2, false), kIdNT, G::CHUNK, G::CHUNK);
          mma_commit(B(G::B_SF));
        }
        if (!wait_bar(B(G::B_DSF), g & 1u, cx.abort_flag)) { ok = false; break; }
        tc_fence_after();
        mma_tn<D>(tm + G::T_DK, tm + G::T_DP, st_desc(m, true), kIdTN, n > 0, acol);
        mma_commit(B(G::B_SLE + m % G::NSLOT));  // Q_n's slot (and its lse2, delta)
        if (n + 1 < T.nb) {
          if (!wait_item(m + 3)) { ok = false; break; }
          tc_fence_after();
          mma_nt<D>(tm + G::T_DP, dv0, st_desc(m + 3, false), kIdNT, G::CHUNK, G::CHUNK);
          mma_commit(B(G::B_DPF));
          if (n + 2 == T.nb) mma_commit(B(G::B_KVE));  // the tile's last read of K and V
        } else {
          mma_commit(B(G::B_ACC));
        }
      }
      m0 += 2u * static_cast<uint32_t>(T.nb);
      g0 += static_cast<uint32_t>(T.nb);
      ++it;
    }
  } else if (warp < 8) {
    // ---- compute: thread = key row r of the tile, warpgroup h = query columns h*64 .. +63
    setmaxnreg_inc<208>();
    const int h = warp >> 2, r = (warp & 3) * 32 + lane;
    const uint32_t tm = cx.tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float c = p.c;
    uint32_t m0 = 0, g0 = 0;
    int it = 0;
    bool ok = true;
    for (int rd = 0; ok && rd * static_cast<int>(gridDim.x) < n_tiles; ++rd) {
      const int t = snake_tile(rd);
      if (t >= n_tiles) continue;
      const KVTile T = kv_tile(p, t);
      const int kv_row0 = T.kt * kBN;
      const int key = kv_row0 + r;
      if (T.nb == 0) {  // no query sees these keys: zero gradients
        if (key < p.Nk) {
          uint16_t* dst = reinterpret_cast<uint16_t*>(h == 0 ? p.dv : p.dk) +
                          (static_cast<size_t>(T.bkv) * p.Nk + key) * D;
          for (int c0 = 0; c0 < D; c0 += 8) *reinterpret_cast<uint4*>(dst + c0) = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      const int nqb = T.nqb;
      for (int n = 0; n < T.nb; ++n) {
        const uint32_t g = g0 + static_cast<uint32_t>(n), m = m0 + 2u * static_cast<uint32_t>(n);
        const int sl = static_cast<int>(m % G::NSLOT);  // the slot of Q_n, with lse2 and delta
        const int i = T.i0 + n % nqb;
        // lse2 / delta of this block were written by the TMA unit: observe its barrier
        ok = wait_bar(B(G::B_SLF + sl), (m / G::NSLOT) & 1u, cx.abort_flag) &&
             wait_bar(B(G::B_SF), g & 1u, cx.abort_flag);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        const float* l2 = reinterpret_cast<const float*>(gbase + G::OFF_SL + sl * G::SLOT_BYTES +
                                                         G::T_BYTES) + h * 64;
        const float* dl = l2 + 128;
        uint32_t sr[64];
        tmem_ld_x64(tm + G::T_S + h * 64, sr);
        // visible query columns of this key row: [lo_c, lo_c + span) -- key k0 + r
        // is seen by query q0 + col iff k0 + r <= q0 + col + wr and k0 + r >= q0 + col - wl
        const int dqk = kv_row0 + r - i * kBM;  // key minus query offset of column 0
        const bool msk = (p.wr >= 0 && kv_row0 + kBN - 1 - p.wr > i * kBM) ||
                         (p.wl >= 0 && kv_row0 + p.wl < i * kBM + kBM - 1);
        const int lo_c = p.wr >= 0 ? dqk - p.wr : -kBM;
        const int hi_c = p.wl >= 0 ? dqk + p.wl : 2 * kBM;
        const uint32_t span = static_cast<uint32_t>(max(hi_c - lo_c + 1, 0));
        // score bias of (query h*64 + x, key r): the tile's row h*64 + x (row 0 if
        // broadcast over queries), 16-bit unit (r % 64) / 8 of box r / 64, rotated
        // by the row (128-byte swizzle)
        const bool rowb = (bias_mode & kBiasRowBcast) != 0;
        if (BIAS) {
          ok = wait_bar(B(G::B_BF), g & 1u, cx.abort_flag);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        }
        const uint32_t bkey = sbase + G::OFF_BIAS + (r >> 6) * (kBiasTileBytes / 2) + (r & 7) * 2;
        const uint32_t bu = static_cast<uint32_t>(r >> 3) & 7u;
        float b_row0 = 0.f;
        if (BIAS && rowb) b_row0 = bias_at(bkey + ((bu ^ 0u) << 4), BF16) * kLog2e;
        float pv[64];
#pragma unroll
        for (int x = 0; x < 64; x += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(l2 + x);
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float bv = 0.f;
            if (BIAS) {
              const uint32_t row = static_cast<uint32_t>(h * 64 + x + e);
              bv = rowb ? b_row0
                        : bias_at(bkey + row * 128u + ((bu ^ static_cast<uint32_t>((x + e) & 7)) << 4), BF16) *
                              kLog2e;
            }
            const float e2 = ex2(fmaf(__uint_as_float(sr[x + e]), c, bv - lv[e]));
            pv[x + e] = (msk && static_cast<uint32_t>(h * 64 + x + e - lo_c) >= span) ? 0.f : e2;
          }
        }
        if (BIAS) {  // this warp has read the bias tile
          __syncwarp();
          if (lane == 0) mbar_arrive(B(G::B_BE));
        }
        uint32_t pk[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) pk[x] = pack2(pv[2 * x], pv[2 * x + 1], BF16);
        tmem_st_x32(tm + G::T_S + h * 64, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(B(G::B_PF));

        ok = wait_bar(B(G::B_DPF), g & 1u, cx.abort_flag);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        uint32_t dr[64];
        tmem_ld_x64(tm + G::T_DP + h * 64, dr);
#pragma unroll
        for (int x = 0; x < 64; x += 4) {
          const float4 d4 = *reinterpret_cast<const float4*>(dl + x);
          const float dv4[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) pv[x + e] *= __uint_as_float(dr[x + e]) - dv4[e];
        }
#pragma unroll
        for (int x = 0; x < 32; ++x) pk[x] = pack2(pv[2 * x], pv[2 * x + 1], BF16);
        tmem_st_x32(tm + G::T_DP + h * 64, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(B(G::B_DSF));
      }
      if (!ok) break;
      // ---- epilogue: warpgroup 0 writes dV, warpgroup 1 writes dK (times scale)
      ok = wait_bar(B(G::B_ACC), static_cast<uint32_t>(it) & 1u, cx.abort_flag);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      const uint32_t m_next = m0 + 2u * static_cast<uint32_t>(T.nb);
      const float mul = h == 0 ? 1.f : p.scale;
      // staging: warpgroup h's four warps in slot (m_next + NSLOT - 2 + h) % NSLOT,
      // 32 rows of D 16-bit values each (16-byte units rotated by the row)
      constexpr int U = D * 2 / 16;  // 16-byte units of a row
      const uint32_t stg = sbase + G::OFF_SL +
                           ((m_next + G::NSLOT - 2 + static_cast<uint32_t>(h)) % G::NSLOT) * G::SLOT_BYTES +
                           static_cast<uint32_t>(warp & 3) * (32u * D * 2u);
      const uint32_t srow = stg + static_cast<uint32_t>(lane) * (D * 2u);
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t a[32];
        tmem_ld_x32(tm + (h == 0 ? G::T_DV : G::T_DK) + c0, a);
        uint32_t w[16];
#pragma unroll
        for (int x = 0; x < 16; ++x)
          w[x] = pack2(__uint_as_float(a[2 * x]) * mul, __uint_as_float(a[2 * x + 1]) * mul, BF16);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const uint32_t u = static_cast<uint32_t>(c0 / 8 + x);
          st_shared_v4(srow + ((u ^ (static_cast<uint32_t>(lane) & (U - 1))) << 4), w + 4 * x);
        }
      }
      // the accumulators are in registers and shared memory: the next tile's
      // first dV and dK may overwrite them
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(B(G::B_ACCE));
      const int key0 = kv_row0 + (warp & 3) * 32;
      uint16_t* out = reinterpret_cast<uint16_t*>(h == 0 ? p.dv : p.dk) +
                      static_cast<size_t>(T.bkv) * p.Nk * D;
#pragma unroll 1
      for (int k = 0; k < U; ++k) {
        const int rr = k * (32 / U) + lane / U, u = lane % U;
        uint32_t w[4];
        ld_shared_v4(stg + static_cast<uint32_t>(rr) * (D * 2u) +
                         ((static_cast<uint32_t>(u) ^ (static_cast<uint32_t>(rr) & (U - 1))) << 4),
                     w);
        if (key0 + rr < p.Nk)
          reinterpret_cast<uint4*>(out + static_cast<size_t>(key0 + rr) * D)[u] =
              make_uint4(w[0], w[1], w[2], w[3]);
      }
      // the TMA unit loads into the staging slots next: order these shared
      // accesses before its writes
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(B(G::B_STG));
      m0 = m_next;
      g0 += static_cast<uint32_t>(T.nb);
      ++it;
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*cx.abort_flag) {  // let issued copies and MMAs land before tensor memory is freed
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) {
    }
  }
  if (threadIdx.x == 0) publish_abort(*cx.abort_flag);
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(cx.tmem, 512);
  }
}

// ================================================================== dQ
template <int D, bool BIAS = false>
struct GeoQ {
  static constexpr int DCH = D / 64;
  static constexpr int T_BYTES = 128 * D * 2;
  static constexpr int CHUNK = 128 * 128;
  // K and V tiles stream through single-tile slots, loaded in the order
  // K0 V0 K1 V1 ...: NKS slots take K_j in turn, NVS slots V_j.  V_j is freed
  // after dP(j), early; K_j only after dQ(j), late -- separate slot sets let
  // V_{j+2} reuse V_j's slot instead of waiting for K_j's.
  // (a score bias takes one K slot's room at head_dim 128 for its tile)
  static constexpr int NSLOT = D == 64 ? 10 : (BIAS ? 4 : 5);
  static constexpr int NVS = D == 64 ? 4 : 2, NKS = NSLOT - NVS;
  // item m (K_{m/2} for even m, V_{m/2} for odd m): its slot, and how many
  // items used that slot before it
  __device__ static int slot(int m) { return (m & 1) ? NKS + (m >> 1) % NVS : (m >> 1) % NKS; }
  __device__ static int use(int m) { return (m & 1) ? (m >> 1) / NVS : (m >> 1) / NKS; }
  static constexpr int OFF_Q = 0, OFF_DO = T_BYTES, OFF_SL = 2 * T_BYTES;
  static constexpr int OFF_BIAS = OFF_SL + NSLOT * T_BYTES;  // the block pair's bias tile
  static constexpr int OFF_BAR = OFF_BIAS + (BIAS ? kBiasTileBytes : 0);
  // (persistent: B_QE = the tile's Q and dO no longer read, B_ACCE = its dQ
  // read out of tensor memory, B_STG = its epilogue done with the staging slot)
  static constexpr int B_QF = 0, B_SLF = 1, B_SLE = 1 + NSLOT, B_SDP = 1 + 2 * NSLOT,
                       B_SFREE = B_SDP + 1, B_DSF = B_SDP + 2, B_DSE = B_SDP + 3, B_DQF = B_SDP + 4,
                       B_BF = B_SDP + 5, B_BE = B_SDP + 6, B_QE = B_SDP + 7, B_ACCE = B_SDP + 8,
                       B_STG = B_SDP + 9, NBAR = B_SDP + 10;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  // TMEM columns: S 0..127, dP 128..255, dS (packed) 256..319, dQ 320..320+D-1
  static constexpr uint32_t T_S = 0, T_DP = 128, T_DS = 256, T_DQ = 320;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(320 + D <= 512, "tensor memory budget");
};

// One query tile of the dQ kernel: (b, query head) row bh, first row q0, its
// key/value head kvz, and the key blocks its rows see, [jb0, jb0 + nb).
struct QTile {
  int bh, q0, kvz, jb0, nb;
};

// tile t: causal launches take the last query blocks (most keys) first
__device__ __forceinline__ QTile q_tile(const BwdParams& p, int t) {
  QTile T;
  const int BH = p.B * p.Hq;
  int qt;
  if (p.causal) {
    qt = p.nqt - 1 - t / BH;
    T.bh = t % BH;
  } else {
    T.bh = t / p.nqt;
    qt = t % p.nqt;
  }
  T.q0 = qt * kBM;
  T.kvz = (T.bh / p.Hq) * p.Hkv + (T.bh % p.Hq) / p.group;
  const int nkb = (p.Nk + kBN - 1) / kBN;
  // key blocks this tile's rows see: keys q - wl .. q + wr (causal: wr = 0)
  const int qlast = min(T.q0 + kBM, p.Nq) - 1;
  T.jb0 = p.wl >= 0 ? min(max(0, T.q0 - p.wl) / kBN, nkb) : 0;
  const int jb1 = p.wr >= 0 ? min(nkb - 1, (qlast + p.wr) / kBN) : nkb - 1;
  T.nb = jb1 >= T.jb0 ? jb1 - T.jb0 + 1 : 0;
  return T;
}

// Persistent like the dK/dV kernel (snake order over the tiles; ring items,
// blocks and tiles counted across tiles): the next tile's Q, dO and first K/V
// blocks load, and its first S and dP run, while the compute warps write the
// previous tile's dQ.  The epilogue stages in the K slot of the next tile's
// NKS-th K block (item M + 2 (NKS - 1), M = the first item after the tile),
// which held the tile's own last K; the TMA thread loads it only after B_STG.
template <int D, bool BF16, bool BIAS = false>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const BwdParams p, const __grid_constant__ CUtensorMap tm_b, const int bias_mode) {
  using G = GeoQ<D, BIAS>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  uint32_t* misc = reinterpret_cast<uint32_t*>(gbase + G::OFF_MISC);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Ctx cx;
  cx.sbase = sbase;
  cx.abort_flag = misc + 1;
  auto B = [&](int i) { return cx.bar(i, G::OFF_BAR); };
  const int n_tiles = p.B * p.Hq * p.nqt;
  constexpr int kGateOff = 2 * (G::NKS - 1);  // staging item, from the first item after a tile

  if (threadIdx.x == 0) {
    mbar_init(B(G::B_QF), 1);
    for (int s = 0; s < G::NSLOT; ++s) {
      mbar_init(B(G::B_SLF + s), 1);
      mbar_init(B(G::B_SLE + s), 1);
    }
    mbar_init(B(G::B_SDP), 1);
    mbar_init(B(G::B_SFREE), 8);
    mbar_init(B(G::B_DSF), 8);
    mbar_init(B(G::B_DSE), 1);
    mbar_init(B(G::B_DQF), 1);
    mbar_init(B(G::B_BF), 1);
    mbar_init(B(G::B_BE), 8);
    mbar_init(B(G::B_QE), 1);
    mbar_init(B(G::B_ACCE), 8);
    mbar_init(B(G::B_STG), 8);
    misc[1] = 0u;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(misc), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cx.tmem = misc[0];

  if (warp >= 8) setmaxnreg_dec<88>();
  if (warp == 9 && lane == 0) {
    // ---- TMA: per tile Q and dO, then (K_j, V_j) per key block
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    const uint64_t pol_first = policy_evict_first(), pol_last = policy_evict_last();
    int m0 = 0;              // ring items issued before this tile
    int gate = -1;           // item that must wait for an epilogue's staging (-1: none)
    uint32_t gate_par = 0;   // ... and that epilogue's B_STG phase
    int it = 0;              // tiles with blocks before this one
    bool ok = true;
    for (int rd = 0; ok && rd * static_cast<int>(gridDim.x) < n_tiles; ++rd) {
      const int t = snake_tile(rd);
      if (t >= n_tiles) continue;
      const QTile T = q_tile(p, t);
      if (T.nb == 0) continue;
      if (it > 0 && !wait_bar(B(G::B_QE), (it - 1) & 1u, cx.abort_flag)) break;
      mbar_arrive_expect_tx(B(G::B_QF), 2 * G::T_BYTES);
#pragma unroll
      for (int c = 0; c < G::DCH; ++c) {
        tma_load_3d(sbase + G::OFF_Q + c * G::CHUNK, &tm_q, B(G::B_QF), c * 64, T.q0, T.bh, pol_first);
        tma_load_3d(sbase + G::OFF_DO + c * G::CHUNK, &tm_do, B(G::B_QF), c * 64, T.q0, T.bh, pol_first);
      }
      for (int mm = 0; mm < 2 * T.nb; ++mm) {  // item mm: K (even) or V (odd) of block mm / 2
        const int m = m0 + mm;
        if (m == gate && !wait_bar(B(G::B_STG), gate_par, cx.abort_flag)) { ok = false; break; }
        const int sl = G::slot(m), u = G::use(m);
        if (u > 0 && !wait_bar(B(G::B_SLE + sl), (u - 1) & 1u, cx.abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(B(G::B_SLF + sl), G::T_BYTES);
#pragma unroll
        for (int c = 0; c < G::DCH; ++c)
          tma_load_3d(sbase + G::OFF_SL + sl * G::T_BYTES + c * G::CHUNK, (mm & 1) ? &tm_v : &tm_k,
                      B(G::B_SLF + sl), c * 64, (T.jb0 + (mm >> 1)) * kBN, T.kvz, pol_last);
      }
      if (!ok) break;
      m0 += 2 * T.nb;
      // a previous epilogue's gate not reached by this tile's items (short
      // tiles): wait for it here, before this tile's gate replaces it
      if (gate >= m0 && !wait_bar(B(G::B_STG), gate_par, cx.abort_flag)) break;
      gate = m0 + kGateOff;
      gate_par = static_cast<uint32_t>(it) & 1u;
      ++it;
    }
  } else if (BIAS && warp == 10 && lane == 0) {
    // ---- TMA: the bias tile of each key block: rows = this tile's queries (one
    // row if broadcast over queries), columns = the block's keys
    const uint64_t pol = policy_evict_last();
    const int rows = (bias_mode & kBiasRowBcast) ? 1 : kBM;
    int g0 = 0;  // blocks before this tile
    bool ok = true;
    for (int rd = 0; ok && rd * static_cast<int>(gridDim.x) < n_tiles; ++rd) {
      const int t = snake_tile(rd);
      if (t >= n_tiles) continue;
      const QTile T = q_tile(p, t);
      if (T.nb == 0) continue;
      for (int j = 0; j < T.nb; ++j) {
        const int g = g0 + j;
        if (g > 0 && !wait_bar(B(G::B_BE), (g - 1) & 1u, cx.abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(B(G::B_BF), 2 * rows * 128);
#pragma unroll
        for (int box = 0; box < 2; ++box)
          tma_load_4d(sbase + G::OFF_BIAS + box * (kBiasTileBytes / 2), &tm_b, B(G::B_BF),
                      (T.jb0 + j) * kBN + box * 64, (bias_mode & kBiasRowBcast) ? 0 : T.q0,
                      (bias_mode & kBiasPerHead) ? T.bh % p.Hq : 0,
                      (bias_mode & kBiasPerBatch) ? T.bh / p.Hq : 0, pol);
      }
      g0 += T.nb;
    }
  } else if (warp == 8 && lane == 0) {
    // ---- MMA, per tile: S(0) dP(0) | S(j+1) dP(j+1) dQ(j) | ...
    constexpr uint32_t kIdNT = idesc_f16(128, 128, BF16, false);
    constexpr uint32_t kIdTN = idesc_f16(128, D, BF16, true);
    const uint32_t tm = cx.tmem;
    const uint64_t dq0 = sdesc_sw128(sbase + G::OFF_Q, 16, 1024);
    const uint64_t ddo0 = sdesc_sw128(sbase + G::OFF_DO, 16, 1024);
    // ring item m (a K or V block): its slot, and the parity of its fill
    auto kv_desc = [&](int m, bool mn) {
      const uint32_t a = sbase + G::OFF_SL + G::slot(m) * G::T_BYTES;
      return mn ? sdesc_sw128(a, G::CHUNK, 1024) : sdesc_sw128(a, 16, 1024);
    };
    auto wait_item = [&](int m) {
      return wait_bar(B(G::B_SLF + G::slot(m)), G::use(m) & 1u, cx.abort_flag);
    };
    // S and dP of the block whose K is item m; its V's slot is free once dP completes
    auto issue_sdp = [&](int m) {
      mma_nt<D>(tm + G::T_S, dq0, kv_desc(m, false), kIdNT, G::CHUNK, G::CHUNK);
      mma_nt<D>(tm + G::T_DP, ddo0, kv_desc(m + 1, false), kIdNT, G::CHUNK, G::CHUNK);
      mma_commit(B(G::B_SDP));
      mma_commit(B(G::B_SLE + G::slot(m + 1)));
    };
    // dS of key column k: warpgroup k / 64 packed its half at columns (k / 64) * 32 ..
    auto acol = [](int kk) { return static_cast<uint32_t>(kk * 8); };
    int m0 = 0, g0 = 0, it = 0;
    bool ok = true;
    for (int rd = 0; ok && rd * static_cast<int>(gridDim.x) < n_tiles; ++rd) {
      const int t = snake_tile(rd);
      if (t >= n_tiles) continue;
      const QTile T = q_tile(p, t);
      if (T.nb == 0) continue;
      // S(0) and dP(0) overwrite S and dP: the compute warps must have read the
      // previous tile's last block
      ok = (g0 == 0 || wait_bar(B(G::B_SFREE), (g0 - 1) & 1u, cx.abort_flag)) &&
           wait_bar(B(G::B_QF), static_cast<uint32_t>(it) & 1u, cx.abort_flag) && wait_item(m0) &&
           wait_item(m0 + 1);
      if (!ok) break;
      tc_fence_after();
      issue_sdp(m0);
      if (T.nb == 1) mma_commit(B(G::B_QE));
      for (int j = 0; j < T.nb; ++j) {
        const int g = g0 + j, m = m0 + 2 * j;
        if (j + 1 < T.nb) {  // next S and dP once the compute warps have read this block's
          if (!wait_bar(B(G::B_SFREE), g & 1u, cx.abort_flag)) { ok = false; break; }
          if (!wait_item(m + 2) || !wait_item(m + 3)) { ok = false; break; }
          tc_fence_after();
          issue_sdp(m + 2);
          if (j + 2 == T.nb) mma_commit(B(G::B_QE));  // the tile's last read of Q and dO
        }
        if (!wait_bar(B(G::B_DSF), g & 1u, cx.abort_flag)) { ok = false; break; }
        // the first dQ of a tile overwrites the accumulator: the previous tile's
        // epilogue must have read it out
        if (j == 0 && it > 0 && !wait_bar(B(G::B_ACCE), (it - 1) & 1u, cx.abort_flag)) { ok = false; break; }
        tc_fence_after();
        mma_tn<D>(tm + G::T_DQ, tm + G::T_DS, kv_desc(m, true), kIdTN, j > 0, acol);
        mma_commit(B(G::B_DSE));
        mma_commit(B(G::B_SLE + G::slot(m)));  // K_j's slot
        if (j + 1 == T.nb) mma_commit(B(G::B_DQF));
      }
      m0 += 2 * T.nb;
      g0 += T.nb;
      ++it;
    }
  } else if (warp < 8) {
    // ---- compute: thread = query row r, warpgroup h = key columns h*64 .. +63
    setmaxnreg_inc<208>();
    // the dK/dV kernel (and before it the prep kernel that wrote lse2 and delta)
    // may still be running (programmatic launch); Q, K, V, dO are inputs, so only
    // these warps wait
    grid_dep_wait();
    const int h = warp >> 2, r = (warp & 3) * 32 + lane;
    const uint32_t tm = cx.tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float c = p.c;
    int m0 = 0, g0 = 0, it = 0;
    bool ok = true;
    for (int rd = 0; ok && rd * static_cast<int>(gridDim.x) < n_tiles; ++rd) {
      const int t = snake_tile(rd);
      if (t >= n_tiles) continue;
      const QTile T = q_tile(p, t);
      const int qpos = T.q0 + r;
      if (T.nb == 0) {  // no key seen by this tile's rows (key windows): dQ = 0
        if (qpos < p.Nq) {
          uint16_t* dst = reinterpret_cast<uint16_t*>(p.dq) + (static_cast<size_t>(T.bh) * p.Nq + qpos) * D;
          for (int c0 = h * (D / 2); c0 < (h + 1) * (D / 2); c0 += 8)
            *reinterpret_cast<uint4*>(dst + c0) = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      const size_t srow = static_cast<size_t>(T.bh) * p.Nq_pad + qpos;
      const float lse2 = __ldcg(p.lse2 + srow), dlt = __ldcg(p.delta + srow);
      for (int j = 0; j < T.nb; ++j) {
        const int g = g0 + j;
        ok = wait_bar(B(G::B_SDP), g & 1u, cx.abort_flag);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[64], dr[64];
        tmem_ld_x64(tm + G::T_S + h * 64, sr);
        tmem_ld_x64(tm + G::T_DP + h * 64, dr);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(B(G::B_SFREE));
        // visible keys of this row in the block: [0, lim)
        const int kbase = (T.jb0 + j) * kBN + h * 64;
        int lim = p.Nk - kbase;  // keys [lo, lim) of this half block are visible to the row
        if (p.wr >= 0) lim = min(lim, qpos + p.wr - kbase + 1);
        const int lo = p.wl >= 0 ? qpos - p.wl - kbase : 0;
        const uint32_t span = static_cast<uint32_t>(max(lim - lo, 0));
        // score bias of this row, keys h*64 .. +63: box h of the tile, row r (row 0
        // if broadcast over queries), 16-byte units rotated by the row
        uint32_t bw[32];
        if (BIAS) {
          ok = wait_bar(B(G::B_BF), g & 1u, cx.abort_flag);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          const uint32_t brow = (bias_mode & kBiasRowBcast) ? 0u : static_cast<uint32_t>(r);
          const uint32_t bb = sbase + G::OFF_BIAS + h * (kBiasTileBytes / 2) + brow * 128u;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(bw[4 * u]), "=r"(bw[4 * u + 1]), "=r"(bw[4 * u + 2]), "=r"(bw[4 * u + 3])
                         : "r"(bb + ((static_cast<uint32_t>(u) ^ (brow & 7u)) << 4)));
          __syncwarp();
          if (lane == 0) mbar_arrive(B(G::B_BE));
        }
        uint32_t pk[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          float2 b2 = make_float2(0.f, 0.f);
          if (BIAS) b2 = unpack2(bw[x], BF16);
          float v2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int i = 2 * x + e;
            const float bv = BIAS ? (e ? b2.y : b2.x) * kLog2e : 0.f;
            const float pe = ex2(fmaf(__uint_as_float(sr[i]), c, bv - lse2));
            v2[e] = static_cast<uint32_t>(i - lo) < span ? pe * (__uint_as_float(dr[i]) - dlt) : 0.f;
          }
          pk[x] = pack2(v2[0], v2[1], BF16);
        }
        if (g > 0) {  // the previous dQ MMA has read the previous dS
          ok = wait_bar(B(G::B_DSE), (g - 1) & 1u, cx.abort_flag);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
        }
        tmem_st_x32(tm + G::T_DS + h * 32, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(B(G::B_DSF));
      }
      if (!ok) break;
      // ---- epilogue: dQ = scale * acc, warpgroup h writes columns h * D/2 .. +D/2
      ok = wait_bar(B(G::B_DQF), static_cast<uint32_t>(it) & 1u, cx.abort_flag);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      const int m_next = m0 + 2 * T.nb;
      // staging: the slot of item m_next + kGateOff; each warp 32 half rows
      // (16-byte units rotated by the row)
      constexpr int U = D / 16;  // 16-byte units of a half row
      const uint32_t stg = sbase + G::OFF_SL + G::slot(m_next + kGateOff) * G::T_BYTES +
                           static_cast<uint32_t>(warp) * (32u * D);
      const uint32_t srow_s = stg + static_cast<uint32_t>(lane) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D / 2; c0 += 32) {
        uint32_t a[32];
        tmem_ld_x32(tm + G::T_DQ + h * (D / 2) + c0, a);
        uint32_t w[16];
#pragma unroll
        for (int x = 0; x < 16; ++x)
          w[x] = pack2(__uint_as_float(a[2 * x]) * p.scale, __uint_as_float(a[2 * x + 1]) * p.scale, BF16);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const uint32_t u = static_cast<uint32_t>(c0 / 8 + x);
          st_shared_v4(srow_s + ((u ^ (static_cast<uint32_t>(lane) & (U - 1))) << 4), w + 4 * x);
        }
      }
      // dQ is in registers and shared memory: the next tile's first dQ may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(B(G::B_ACCE));
      const int q0w = T.q0 + (warp & 3) * 32;
      uint16_t* out = reinterpret_cast<uint16_t*>(p.dq) + static_cast<size_t>(T.bh) * p.Nq * D + h * (D / 2);
#pragma unroll 1
      for (int k = 0; k < U; ++k) {
        const int rr = k * (32 / U) + lane / U, u = lane % U;
        uint32_t w[4];
        ld_shared_v4(stg + static_cast<uint32_t>(rr) * D +
                         ((static_cast<uint32_t>(u) ^ (static_cast<uint32_t>(rr) & (U - 1))) << 4),
                     w);
        if (q0w + rr < p.Nq)
          reinterpret_cast<uint4*>(out + static_cast<size_t>(q0w + rr) * D)[u] =
              make_uint4(w[0], w[1], w[2], w[3]);
      }
      // the TMA unit loads into the staging slot next: order these shared
      // accesses before its writes
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(B(G::B_STG));
      m0 = m_next;
      g0 += T.nb;
      ++it;
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*cx.abort_flag) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) {
    }
  }
  if (threadIdx.x == 0) publish_abort(*cx.abort_flag);
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(cx.tmem, 512);
  }
}


// ================================================================== head_dim 256
// At D = 256 one CTA cannot keep what the kernels above keep on chip: dK and
// dV alone fill the 512 tensor-memory columns, and 128-row K, V, Q and dO
// tiles are 64 KB each.  So here
//   * the streamed operand comes in blocks of 64 rows (query blocks in the
//     key-tile kernels, key blocks in the dQ kernel), 32 KB each;
//   * dV and dK come from two launches of one key-tile kernel, each with a
//     single 256-column accumulator:
//       DK = false:  S^T = K Q^T, P^T, dV += P^T dO
//       DK = true:   S^T = K Q^T, dP^T = V dO^T, dS^T, dK += dS^T Q
//     (S^T is formed in both: one extra MMA group per block pair);
//   * bwd_dq256_kernel: S = Q K^T, dP = dO V^T, dS, dQ += dS K.
// The blocks stream through two sets of slots: one for the operand held until
// the block's last MMA (Q in the key-tile kernels, K in dQ), one for the
// operand released early (dO after dP^T or dV; V after dP).
constexpr int kBS = 64;  // rows of a streamed block at head_dim 256

// Accumulating MMA over KSTEPS steps of 16 along K, A (16-bit) in tensor
// memory at column acol(kk), B an MN-major SW128 block (16 rows of K per step).
template <int KSTEPS, typename ACol>
__device__ __forceinline__ void mma_tn_steps(uint32_t d, uint32_t a, uint64_t b0, uint32_t idesc,
                                             bool acc, ACol acol) {
#pragma unroll
  for (int kk = 0; kk < KSTEPS; ++kk)
    mma_ts(d, a + acol(kk), b0 + static_cast<uint64_t>((kk * 2048) >> 4), idesc,
           (acc || kk > 0) ? 1u : 0u);
}

struct Geo256 {
  static constexpr int CH_R = 128 * 128;   // one 64-column chunk of a 128-row tile
  static constexpr int CH_S = kBS * 128;   // one 64-column chunk of a 64-row block
  static constexpr int TILE_R = 4 * CH_R;  // 64 KB
  static constexpr int TILE_S = 4 * CH_S;  // 32 KB
};

template <bool DK>
struct Geo256KV : Geo256 {
  // slot sets: NA for Q blocks (with their lse2 and delta), NB for dO blocks;
  // item m is Q_{m/2} (even) or dO_{m/2} (odd)
  static constexpr int NA = DK ? 2 : 3, NB = DK ? 1 : 2, NSLOT = NA + NB;
  __device__ static int slot(int m) { return (m & 1) ? NA + (m >> 1) % NB : (m >> 1) % NA; }
  __device__ static int use(int m) { return (m & 1) ? (m >> 1) / NB : (m >> 1) / NA; }
  static constexpr int OFF_K = 0, OFF_V = TILE_R, OFF_SL = DK ? 2 * TILE_R : TILE_R;
  static constexpr int OFF_SIDE = OFF_SL + NSLOT * TILE_S;  // per Q slot: lse2[64], delta[64]
  static constexpr int OFF_BAR = OFF_SIDE + NA * 512;
  static constexpr int B_KV = 0, B_SLF = 1, B_SLE = 1 + NSLOT, B_SF = 1 + 2 * NSLOT,
                       B_DPF = B_SF + 1, B_PF = B_SF + 2, B_ACC = B_SF + 3, NBAR = B_SF + 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  // TMEM columns: S^T 0..63 (P^T packed over it), dP^T 64..127 (dS^T packed
  // over it), the accumulator (dV or dK) 256..511
  static constexpr uint32_t TM_S = 0, TM_DP = 64, TM_ACC = 256;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <bool BF16, bool DK>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kv256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const BwdParams p) {
  using G = Geo256KV<DK>;
  constexpr int D = 256;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  uint32_t* misc = reinterpret_cast<uint32_t*>(gbase + G::OFF_MISC);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Ctx cx;
  cx.sbase = sbase;
  cx.abort_flag = misc + 1;
  auto B = [&](int i) { return cx.bar(i, G::OFF_BAR); };
  const KVTile T = kv_tile(p, blockIdx.x, kBS);

  if (threadIdx.x == 0) {
    mbar_init(B(G::B_KV), 1);
    for (int s = 0; s < G::NSLOT; ++s) {
      mbar_init(B(G::B_SLF + s), 1);
      mbar_init(B(G::B_SLE + s), 1);
    }
    mbar_init(B(G::B_SF), 1);
    mbar_init(B(G::B_DPF), 1);
    mbar_init(B(G::B_PF), 8);
    mbar_init(B(G::B_ACC), 1);
    misc[1] = 0u;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(misc), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cx.tmem = misc[0];

  // Registers: 176 for the compute warpgroups (32 scores a thread per block),
  // 152 for the rest, whose MMA groups run 16 steps of K (2 x 128 x 176 +
  // 128 x 152 = 384 x 168).
  const int kv_row0 = T.kt * kBN;
  const int nqb = T.nqb;
  if (warp >= 8) setmaxnreg_dec<152>();
  if (warp == 9 && lane == 0 && T.nb > 0) {
    // ---- TMA: K (and V) once, then (Q + lse2 [+ delta], dO) per 64-row query block
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_do);
    const uint64_t pol_first = policy_evict_first(), pol_last = policy_evict_last();
    mbar_arrive_expect_tx(B(G::B_KV), (DK ? 2 : 1) * G::TILE_R);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      tma_load_3d(sbase + G::OFF_K + c * G::CH_R, &tm_k, B(G::B_KV), c * 64, kv_row0, T.bkv, pol_first);
      if (DK)
        tma_load_3d(sbase + G::OFF_V + c * G::CH_R, &tm_v, B(G::B_KV), c * 64, kv_row0, T.bkv,
                    pol_first);
    }
    for (int m = 0; m < 2 * T.nb; ++m) {
      const int sl = G::slot(m), u = G::use(m), n = m >> 1;
      if (u > 0 && !wait_bar(B(G::B_SLE + sl), (u - 1) & 1u, cx.abort_flag)) break;
      const int h = n / nqb, i = T.i0 + n % nqb;
      const int bh = (T.bkv / p.Hkv) * p.Hq + (T.bkv % p.Hkv) * p.group + h;
      const bool is_q = (m & 1) == 0;
      mbar_arrive_expect_tx(B(G::B_SLF + sl), G::TILE_S + (is_q ? (DK ? 512 : 256) : 0));
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tma_load_3d(sbase + G::OFF_SL + sl * G::TILE_S + c * G::CH_S, is_q ? &tm_q : &tm_do,
                    B(G::B_SLF + sl), c * 64, i * kBS, bh, pol_last);
      if (is_q) {
        const size_t row = static_cast<size_t>(bh) * p.Nq_pad + static_cast<size_t>(i) * kBS;
        const uint32_t side = sbase + G::OFF_SIDE + sl * 512;
        bulk_load(side, p.lse2 + row, 256, B(G::B_SLF + sl));
        if (DK) bulk_load(side + 256, p.delta + row, 256, B(G::B_SLF + sl));
      }
    }
  } else if (warp == 8 && lane == 0 && T.nb > 0) {
    // ---- MMA.  dV: S^T(0) | dV(n) S^T(n+1) | ...;  dK: S^T(0) dP^T(0) | dK(n) S^T(n+1) dP^T(n+1) | ...
    constexpr uint32_t kIdNT = idesc_f16(128, kBS, BF16, false);
    constexpr uint32_t kIdTN = idesc_f16(128, D, BF16, true);
    const uint32_t tm = cx.tmem;
    const uint64_t dk0 = sdesc_sw128(sbase + G::OFF_K, 16, 1024);
    const uint64_t dv0 = sdesc_sw128(sbase + G::OFF_V, 16, 1024);
    auto st_desc = [&](int m, bool mn) {
      const uint32_t a = sbase + G::OFF_SL + G::slot(m) * G::TILE_S;
      return mn ? sdesc_sw128(a, G::CH_S, 1024) : sdesc_sw128(a, 16, 1024);
    };
    auto wait_item = [&](int m) {
      return wait_bar(B(G::B_SLF + G::slot(m)), G::use(m) & 1u, cx.abort_flag);
    };
    // P^T / dS^T of query column x: warpgroup x / 32 packed its 32 columns into
    // its own first 16 -> K step kk (16 queries) at (kk / 2) * 32 + (kk % 2) * 8
    auto acol = [](int kk) { return static_cast<uint32_t>((kk >> 1) * 32 + (kk & 1) * 8); };
    auto issue_s = [&](int n) {  // S^T(n), and dP^T(n) for dK (dO_n's slot is then free)
      mma_nt<D>(tm + G::TM_S, dk0, st_desc(2 * n, false), kIdNT, G::CH_R, G::CH_S);
      mma_commit(B(G::B_SF));
      if (DK) {
        mma_nt<D>(tm + G::TM_DP, dv0, st_desc(2 * n + 1, false), kIdNT, G::CH_R, G::CH_S);
        mma_commit(B(G::B_DPF));
        mma_commit(B(G::B_SLE + G::slot(2 * n + 1)));
      }
    };
    bool ok = wait_bar(B(G::B_KV), 0u, cx.abort_flag) && wait_item(0) && (!DK || wait_item(1));
    if (ok) {
      tc_fence_after();
      issue_s(0);
    }
    for (int n = 0; ok && n < T.nb; ++n) {
      if (!wait_bar(B(G::B_PF), n & 1u, cx.abort_flag)) break;
      if (!DK && !wait_item(2 * n + 1)) break;
      tc_fence_after();
      if (DK) {  // dK += dS^T Q_n
        mma_tn_steps<kBS / 16>(tm + G::TM_ACC, tm + G::TM_DP, st_desc(2 * n, true), kIdTN, n > 0, acol);
      } else {  // dV += P^T dO_n
        mma_tn_steps<kBS / 16>(tm + G::TM_ACC, tm + G::TM_S, st_desc(2 * n + 1, true), kIdTN, n > 0, acol);
        mma_commit(B(G::B_SLE + G::slot(2 * n + 1)));
      }
      mma_commit(B(G::B_SLE + G::slot(2 * n)));  // Q_n's slot (and its lse2, delta)
      if (n + 1 < T.nb) {
        if (!wait_item(2 * n + 2) || (DK && !wait_item(2 * n + 3))) break;
        tc_fence_after();
        issue_s(n + 1);
      } else {
        mma_commit(B(G::B_ACC));
      }
    }
  } else if (warp < 8) {
    // ---- compute: thread = key row r of the tile, warpgroup h = query columns h*32 .. +31
    setmaxnreg_inc<176>();
    const int h = warp >> 2, r = (warp & 3) * 32 + lane;
    const uint32_t tm = cx.tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float c = p.c;
    bool ok = true;
    for (int n = 0; ok && n < T.nb; ++n) {
      const int sl = G::slot(2 * n);  // the slot of Q_n, with lse2 and delta
      const int i = T.i0 + n % nqb;
      // lse2 / delta of this block were written by the TMA unit: observe its barrier
      ok = wait_bar(B(G::B_SLF + sl), G::use(2 * n) & 1u, cx.abort_flag) &&
           wait_bar(B(G::B_SF), n & 1u, cx.abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const float* l2 = reinterpret_cast<const float*>(gbase + G::OFF_SIDE + sl * 512) + h * 32;
      const float* dl = l2 + 64;
      uint32_t sr[32];
      tmem_ld_x32(tm + G::TM_S + h * 32, sr);
      // visible query columns of this key row: [lo_c, lo_c + span) -- key k0 + r
      // is seen by query q0 + col iff k0 + r <= q0 + col + wr and k0 + r >= q0 + col - wl
      const int q0 = i * kBS;
      const int dqk = kv_row0 + r - q0;
      const bool msk = (p.wr >= 0 && kv_row0 + kBN - 1 - p.wr > q0) ||
                       (p.wl >= 0 && kv_row0 + p.wl < q0 + kBS - 1);
      const int lo_c = p.wr >= 0 ? dqk - p.wr : -kBN;
      const int hi_c = p.wl >= 0 ? dqk + p.wl : kBN + kBS;
      const uint32_t span = static_cast<uint32_t>(max(hi_c - lo_c + 1, 0));
      float pv[32];
#pragma unroll
      for (int x = 0; x < 32; x += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(l2 + x);
        const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float e2 = ex2(fmaf(__uint_as_float(sr[x + e]), c, -lv[e]));
          pv[x + e] = (msk && static_cast<uint32_t>(h * 32 + x + e - lo_c) >= span) ? 0.f : e2;
        }
      }
      uint32_t pk[16];
      if (DK) {  // dS^T = P^T (dP^T - Delta), over dP^T
        ok = wait_bar(B(G::B_DPF), n & 1u, cx.abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
        uint32_t dr[32];
        tmem_ld_x32(tm + G::TM_DP + h * 32, dr);
#pragma unroll
        for (int x = 0; x < 32; x += 4) {
          const float4 d4 = *reinterpret_cast<const float4*>(dl + x);
          const float dv4[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) pv[x + e] *= __uint_as_float(dr[x + e]) - dv4[e];
        }
#pragma unroll
        for (int x = 0; x < 16; ++x) pk[x] = pack2(pv[2 * x], pv[2 * x + 1], BF16);
        tmem_st_x16(tm + G::TM_DP + h * 32, pk);
      } else {  // P^T, over S^T
#pragma unroll
        for (int x = 0; x < 16; ++x) pk[x] = pack2(pv[2 * x], pv[2 * x + 1], BF16);
        tmem_st_x16(tm + G::TM_S + h * 32, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(B(G::B_PF));
    }
    // ---- epilogue: warpgroup h writes columns h*128 .. +127 of dV, or of dK (times scale)
    const int key = kv_row0 + r;
    uint16_t* dst = reinterpret_cast<uint16_t*>(DK ? p.dk : p.dv) +
                    (static_cast<size_t>(T.bkv) * p.Nk + (key < p.Nk ? key : 0)) * D;
    const float mul = DK ? p.scale : 1.f;
    if (T.nb == 0) {  // no query sees these keys: zero gradients
      if (key < p.Nk)
        for (int c0 = h * 128; c0 < (h + 1) * 128; c0 += 8)
          *reinterpret_cast<uint4*>(dst + c0) = make_uint4(0, 0, 0, 0);
    } else if (ok) {
      ok = wait_bar(B(G::B_ACC), 0u, cx.abort_flag);
      if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
#pragma unroll 1
        for (int c0 = h * 128; c0 < (h + 1) * 128; c0 += 32) {
          uint32_t a[32];
          tmem_ld_x32(tm + G::TM_ACC + c0, a);
          uint32_t w[16];
#pragma unroll
          for (int x = 0; x < 16; ++x)
            w[x] = pack2(__uint_as_float(a[2 * x]) * mul, __uint_as_float(a[2 * x + 1]) * mul, BF16);
          if (key < p.Nk) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
            for (int x = 0; x < 4; ++x) d4[x] = make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
          }
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*cx.abort_flag) {  // let issued copies and MMAs land before tensor memory is freed
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) {
    }
  }
  if (threadIdx.x == 0) publish_abort(*cx.abort_flag);
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(cx.tmem, 512);
  }
}

struct Geo256Q : Geo256 {
  // slot sets: NA for K blocks (held until dQ), NB for V blocks (free after dP);
  // item m is K_{m/2} (even) or V_{m/2} (odd)
  static constexpr int NA = 2, NB = 1, NSLOT = NA + NB;
  __device__ static int slot(int m) { return (m & 1) ? NA + (m >> 1) % NB : (m >> 1) % NA; }
  __device__ static int use(int m) { return (m & 1) ? (m >> 1) / NB : (m >> 1) / NA; }
  static constexpr int OFF_Q = 0, OFF_DO = TILE_R, OFF_SL = 2 * TILE_R;
  static constexpr int OFF_BAR = OFF_SL + NSLOT * TILE_S;
  static constexpr int B_QF = 0, B_SLF = 1, B_SLE = 1 + NSLOT, B_SDP = 1 + 2 * NSLOT,
                       B_SFREE = B_SDP + 1, B_DSF = B_SDP + 2, B_DSE = B_SDP + 3, B_DQF = B_SDP + 4,
                       NBAR = B_SDP + 5;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  // TMEM columns: S 0..63, dP 64..127, dS (packed) 128..159, dQ 256..511
  static constexpr uint32_t TM_S = 0, TM_DP = 64, TM_DS = 128, TM_DQ = 256;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const BwdParams p) {
  using G = Geo256Q;
  constexpr int D = 256;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  uint32_t* misc = reinterpret_cast<uint32_t*>(gbase + G::OFF_MISC);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Ctx cx;
  cx.sbase = sbase;
  cx.abort_flag = misc + 1;
  auto B = [&](int i) { return cx.bar(i, G::OFF_BAR); };

  // tile: (b, hq, 128-row query block); causal: the last query blocks (most keys) first
  const int BH = p.B * p.Hq, t = blockIdx.x;
  int bh, qt;
  if (p.causal) {
    qt = p.nqt - 1 - t / BH;
    bh = t % BH;
  } else {
    bh = t / p.nqt;
    qt = t % p.nqt;
  }
  const int q0 = qt * kBM;
  const int kvz = (bh / p.Hq) * p.Hkv + (bh % p.Hq) / p.group;
  const int nkb = (p.Nk + kBS - 1) / kBS;
  // 64-key blocks this tile's rows see: keys q - wl .. q + wr (causal: wr = 0)
  const int qlast = min(q0 + kBM, p.Nq) - 1;
  const int jb0 = p.wl >= 0 ? min(max(0, q0 - p.wl) / kBS, nkb) : 0;
  const int jb1 = p.wr >= 0 ? min(nkb - 1, (qlast + p.wr) / kBS) : nkb - 1;
  const int nb = jb1 >= jb0 ? jb1 - jb0 + 1 : 0;

  if (threadIdx.x == 0) {
    mbar_init(B(G::B_QF), 1);
    for (int s = 0; s < G::NSLOT; ++s) {
      mbar_init(B(G::B_SLF + s), 1);
      mbar_init(B(G::B_SLE + s), 1);
    }
    mbar_init(B(G::B_SDP), 1);
    mbar_init(B(G::B_SFREE), 8);
    mbar_init(B(G::B_DSF), 8);
    mbar_init(B(G::B_DSE), 1);
    mbar_init(B(G::B_DQF), 1);
    misc[1] = 0u;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(misc), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cx.tmem = misc[0];

  // Registers: as in bwd_kv256_kernel (176 / 152).
  if (warp >= 8) setmaxnreg_dec<152>();
  if (warp == 9 && lane == 0 && nb > 0) {
    // ---- TMA: Q and dO once, then (K_j, V_j) per 64-key block
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    const uint64_t pol_first = policy_evict_first(), pol_last = policy_evict_last();
    mbar_arrive_expect_tx(B(G::B_QF), 2 * G::TILE_R);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      tma_load_3d(sbase + G::OFF_Q + c * G::CH_R, &tm_q, B(G::B_QF), c * 64, q0, bh, pol_first);
      tma_load_3d(sbase + G::OFF_DO + c * G::CH_R, &tm_do, B(G::B_QF), c * 64, q0, bh, pol_first);
    }
    for (int m = 0; m < 2 * nb; ++m) {
      const int sl = G::slot(m), u = G::use(m);
      if (u > 0 && !wait_bar(B(G::B_SLE + sl), (u - 1) & 1u, cx.abort_flag)) break;
      mbar_arrive_expect_tx(B(G::B_SLF + sl), G::TILE_S);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tma_load_3d(sbase + G::OFF_SL + sl * G::TILE_S + c * G::CH_S, (m & 1) ? &tm_v : &tm_k,
                    B(G::B_SLF + sl), c * 64, (jb0 + (m >> 1)) * kBS, kvz, pol_last);
    }
  } else if (warp == 8 && lane == 0 && nb > 0) {
    // ---- MMA: S(0) dP(0) | S(j+1) dP(j+1) dQ(j) | ...
    constexpr uint32_t kIdNT = idesc_f16(128, kBS, BF16, false);
    constexpr uint32_t kIdTN = idesc_f16(128, D, BF16, true);
    const uint32_t tm = cx.tmem;
    const uint64_t dq0 = sdesc_sw128(sbase + G::OFF_Q, 16, 1024);
    const uint64_t ddo0 = sdesc_sw128(sbase + G::OFF_DO, 16, 1024);
    auto kv_desc = [&](int m, bool mn) {
      const uint32_t a = sbase + G::OFF_SL + G::slot(m) * G::TILE_S;
      return mn ? sdesc_sw128(a, G::CH_S, 1024) : sdesc_sw128(a, 16, 1024);
    };
    auto wait_item = [&](int m) {
      return wait_bar(B(G::B_SLF + G::slot(m)), G::use(m) & 1u, cx.abort_flag);
    };
    auto issue_sdp = [&](int j) {  // S(j), dP(j); V_j's slot is free once dP(j) completes
      mma_nt<D>(tm + G::TM_S, dq0, kv_desc(2 * j, false), kIdNT, G::CH_R, G::CH_S);
      mma_nt<D>(tm + G::TM_DP, ddo0, kv_desc(2 * j + 1, false), kIdNT, G::CH_R, G::CH_S);
      mma_commit(B(G::B_SDP));
      mma_commit(B(G::B_SLE + G::slot(2 * j + 1)));
    };
    // dS of key column x: warpgroup x / 32 packed its 32 columns at 16 * (x / 32) ..
    auto acol = [](int kk) { return static_cast<uint32_t>(kk * 8); };
    bool ok = wait_bar(B(G::B_QF), 0u, cx.abort_flag) && wait_item(0) && wait_item(1);
    if (ok) {
      tc_fence_after();
      issue_sdp(0);
    }
    for (int j = 0; ok && j < nb; ++j) {
      if (j + 1 < nb) {  // next S and dP once the compute warps have read this block's
        if (!wait_bar(B(G::B_SFREE), j & 1u, cx.abort_flag)) break;
        if (!wait_item(2 * j + 2) || !wait_item(2 * j + 3)) break;
        tc_fence_after();
        issue_sdp(j + 1);
      }
      if (!wait_bar(B(G::B_DSF), j & 1u, cx.abort_flag)) break;
      tc_fence_after();
      mma_tn_steps<kBS / 16>(tm + G::TM_DQ, tm + G::TM_DS, kv_desc(2 * j, true), kIdTN, j > 0, acol);
      mma_commit(B(G::B_DSE));
      mma_commit(B(G::B_SLE + G::slot(2 * j)));  // K_j's slot
      if (j + 1 == nb) mma_commit(B(G::B_DQF));
    }
  } else if (warp < 8) {
    // ---- compute: thread = query row r, warpgroup h = key columns h*32 .. +31
    setmaxnreg_inc<176>();
    const int h = warp >> 2, r = (warp & 3) * 32 + lane;
    const uint32_t tm = cx.tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float c = p.c;
    const size_t srow = static_cast<size_t>(bh) * p.Nq_pad + q0 + r;
    const float lse2 = p.lse2[srow], dlt = p.delta[srow];
    const int qpos = q0 + r;
    bool ok = true;
    for (int j = 0; ok && j < nb; ++j) {
      ok = wait_bar(B(G::B_SDP), j & 1u, cx.abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t sr[32], dr[32];
      tmem_ld_x32(tm + G::TM_S + h * 32, sr);
      tmem_ld_x32(tm + G::TM_DP + h * 32, dr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(B(G::B_SFREE));
      // visible keys of this row in the block half: [lo, lim)
      const int kbase = (jb0 + j) * kBS + h * 32;
      int lim = p.Nk - kbase;
      if (p.wr >= 0) lim = min(lim, qpos + p.wr - kbase + 1);
      const int lo = p.wl >= 0 ? qpos - p.wl - kbase : 0;
      const uint32_t span = static_cast<uint32_t>(max(lim - lo, 0));
      uint32_t pk[16];
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        float v2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int i = 2 * x + e;
          const float pe = ex2(fmaf(__uint_as_float(sr[i]), c, -lse2));
          v2[e] = static_cast<uint32_t>(i - lo) < span ? pe * (__uint_as_float(dr[i]) - dlt) : 0.f;
        }
        pk[x] = pack2(v2[0], v2[1], BF16);
      }
      if (j > 0) {  // dQ(j-1) has read the previous dS
        ok = wait_bar(B(G::B_DSE), (j - 1) & 1u, cx.abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
      }
      tmem_st_x16(tm + G::TM_DS + h * 16, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(B(G::B_DSF));
    }
    // ---- epilogue: dQ = scale * acc, warpgroup h writes columns h*128 .. +127
    if (nb == 0 && qpos < p.Nq) {  // no key seen by this tile's rows (key windows): dQ = 0
      uint16_t* dst = reinterpret_cast<uint16_t*>(p.dq) + (static_cast<size_t>(bh) * p.Nq + qpos) * D;
      for (int c0 = h * 128; c0 < (h + 1) * 128; c0 += 8)
        *reinterpret_cast<uint4*>(dst + c0) = make_uint4(0, 0, 0, 0);
    }
    if (ok && nb > 0) {
      ok = wait_bar(B(G::B_DQF), 0u, cx.abort_flag);
      if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        uint16_t* dst = reinterpret_cast<uint16_t*>(p.dq) +
                        (static_cast<size_t>(bh) * p.Nq + (qpos < p.Nq ? qpos : 0)) * D;
#pragma unroll 1
        for (int c0 = h * 128; c0 < (h + 1) * 128; c0 += 32) {
          uint32_t a[32];
          tmem_ld_x32(tm + G::TM_DQ + c0, a);
          uint32_t w[16];
#pragma unroll
          for (int x = 0; x < 16; ++x)
            w[x] = pack2(__uint_as_float(a[2 * x]) * p.scale, __uint_as_float(a[2 * x + 1]) * p.scale,
                         BF16);
          if (qpos < p.Nq) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
            for (int x = 0; x < 4; ++x) d4[x] = make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
          }
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*cx.abort_flag) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) {
    }
  }
  if (threadIdx.x == 0) publish_abort(*cx.abort_flag);
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(cx.tmem, 512);
  }
}

}  // namespace fab

// ============================================================================ host side
namespace {

using EncodeTiledFnB = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFnB encode_fn_b() {
  static EncodeTiledFnB fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFnB>(f);
  });
  return fn;
}

// [Z][rows][D] 16-bit tensor, 64 x box_rows boxes, 128-byte swizzle, zero fill out of range.
bool map_rows(CUtensorMap* m, const void* ptr, int D, long long rows, long long Z, bool bf16,
              int box_rows = 128) {
  EncodeTiledFnB enc = encode_fn_b();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)Z};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t es[3] = {1u, 1u, 1u};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
             const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A score bias: element (b, hq, i, j) at ptr + b * sb + hq * sh + i * sq + j
// (elements; a zero stride broadcasts that dimension).
struct BiasArgB {
  const void* ptr;
  long long sb, sh, sq;
};

// [B][H][Nq][Nk] view of the bias with broadcast dimensions of extent 1; boxes
// of 64 keys x 128 rows (1 row when broadcast over queries), 128-byte swizzle.
bool map_bias(CUtensorMap* m, const BiasArgB& a, int B, int H, int Nq, int Nk, bool bf16) {
  EncodeTiledFnB enc = encode_fn_b();
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

bool overlaps_b(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

int nq_pad(int Nq) { return (Nq + 127) / 128 * 128; }

// Launch with programmatic stream serialisation: the kernel may start while the
// previous kernel in the stream still runs (once every CTA of that one has
// signalled it, griddepcontrol.launch_dependents); it waits with
// griddepcontrol.wait before it touches what that kernel writes.
template <typename... Params, typename... Args>
cudaError_t launch_after(void (*kern)(Params...), unsigned grid, int smem, cudaStream_t st,
                         Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(fab::kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Parameters shared by the kernels, and the Delta / LSE * log2(e) pass.
template <int D, bool BF16>
int setup_bwd(fab::BwdParams& p, const void* o, const void* dout, const float* lse, void* dq,
              void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nk, float scale, int causal,
              int wl, int wr, cudaStream_t st, void* ws, int sms) {
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.Nq_pad = nq_pad(Nq);
  p.group = Hq / Hkv;
  p.causal = causal ? 1 : 0;
  p.wl = wl;
  p.wr = causal ? 0 : wr;
  p.scale = scale;
  p.c = scale * fab::kLog2e;
  p.nqt = p.Nq_pad / 128;
  p.nkt = (Nk + 127) / 128;
  float* lse2 = static_cast<float*>(ws);
  float* delta = lse2 + (size_t)B * Hq * p.Nq_pad;
  p.lse2 = lse2;
  p.delta = delta;
  const long long rows = (long long)B * Hq * p.Nq_pad;
  const long long warps_needed = (rows * (D / 8) + 32 * fab::kPrepGroups - 1) / (32 * fab::kPrepGroups);
  long long blocks = (warps_needed + 7) / 8;
  if (blocks > 16LL * sms) blocks = 16LL * sms;
  fab::bwd_prep_kernel<D, BF16><<<(unsigned)blocks, 256, 0, st>>>(
      static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), lse, lse2, delta,
      B * Hq, Nq, p.Nq_pad);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

// head_dim 256: dV and dK from two launches of the key-tile kernel (64-row
// query blocks), dQ over 64-key blocks
template <bool BF16>
int launch_bwd256(const void* q, const void* k, const void* v, const void* o, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq,
                  int Nk, float scale, int causal, int wl, int wr, cudaStream_t st, void* ws,
                  int sms) {
  using GV = fab::Geo256KV<false>;
  using GK = fab::Geo256KV<true>;
  using GQ = fab::Geo256Q;
  static std::once_flag once;
  static bool attr_ok = false;
  std::call_once(once, [] {
    attr_ok = cudaFuncSetAttribute(fab::bwd_kv256_kernel<BF16, false>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   GV::SMEM_BYTES) == cudaSuccess &&
              cudaFuncSetAttribute(fab::bwd_kv256_kernel<BF16, true>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   GK::SMEM_BYTES) == cudaSuccess &&
              cudaFuncSetAttribute(fab::bwd_dq256_kernel<BF16>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   GQ::SMEM_BYTES) == cudaSuccess;
  });
  if (!attr_ok) return FA_ERR_LAUNCH;
  constexpr int D = 256;
  // 128-row tiles (resident operands) and 64-row blocks (streamed operands)
  CUtensorMap tq, tdo, tk, tv, tq_s, tdo_s, tk_s, tv_s;
  const long long zq = (long long)B * Hq, zk = (long long)B * Hkv;
  if (!map_rows(&tq, q, D, Nq, zq, BF16) || !map_rows(&tdo, dout, D, Nq, zq, BF16) ||
      !map_rows(&tk, k, D, Nk, zk, BF16) || !map_rows(&tv, v, D, Nk, zk, BF16) ||
      !map_rows(&tq_s, q, D, Nq, zq, BF16, fab::kBS) ||
      !map_rows(&tdo_s, dout, D, Nq, zq, BF16, fab::kBS) ||
      !map_rows(&tk_s, k, D, Nk, zk, BF16, fab::kBS) || !map_rows(&tv_s, v, D, Nk, zk, BF16, fab::kBS))
    return FA_ERR_DRIVER;
  fab::BwdParams p;
  const int rc = setup_bwd<D, BF16>(p, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, scale, causal,
                                    wl, wr, st, ws, sms);
  if (rc != FA_OK) return rc;
  const unsigned kv_grid = (unsigned)(B * Hkv * p.nkt);
  fab::bwd_kv256_kernel<BF16, false><<<kv_grid, fab::kThreads, GV::SMEM_BYTES, st>>>(
      tq_s, tdo_s, tk, tv, p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  fab::bwd_kv256_kernel<BF16, true><<<kv_grid, fab::kThreads, GK::SMEM_BYTES, st>>>(
      tq_s, tdo_s, tk, tv, p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  fab::bwd_dq256_kernel<BF16><<<(unsigned)(B * Hq * p.nqt), fab::kThreads, GQ::SMEM_BYTES, st>>>(
      tq, tdo, tk_s, tv_s, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

template <int D, bool BF16, bool BIAS = false>
int launch_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
               const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq,
               int Nk, float scale, int causal, int wl, int wr, cudaStream_t st, void* ws,
               int sms, const BiasArgB* bias = nullptr) {
  using GK = fab::GeoKV<D, BIAS>;
  using GQ = fab::GeoQ<D, BIAS>;
  static std::once_flag once;
  static bool attr_ok = false;
  std::call_once(once, [] {
    attr_ok = cudaFuncSetAttribute(fab::bwd_dkdv_kernel<D, BF16, BIAS>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   GK::SMEM_BYTES) == cudaSuccess &&
              cudaFuncSetAttribute(fab::bwd_dq_kernel<D, BF16, BIAS>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   GQ::SMEM_BYTES) == cudaSuccess;
  });
  if (!attr_ok) return FA_ERR_LAUNCH;
  CUtensorMap tq, tdo, tk, tv;
  if (!map_rows(&tq, q, D, Nq, (long long)B * Hq, BF16) ||
      !map_rows(&tdo, dout, D, Nq, (long long)B * Hq, BF16) ||
      !map_rows(&tk, k, D, Nk, (long long)B * Hkv, BF16) ||
      !map_rows(&tv, v, D, Nk, (long long)B * Hkv, BF16))
    return FA_ERR_DRIVER;
  CUtensorMap tb = tk;  // (unused without a bias)
  int bias_mode = 0;
  if (BIAS) {
    if (!map_bias(&tb, *bias, B, Hq, Nq, Nk, BF16)) return FA_ERR_DRIVER;
    bias_mode = (bias->sq ? 0 : fab::kBiasRowBcast) | (bias->sh ? fab::kBiasPerHead : 0) |
                (bias->sb ? fab::kBiasPerBatch : 0);
  }
  // 1. Delta and LSE * log2(e), padded
  fab::BwdParams p;
  const int rc = setup_bwd<D, BF16>(p, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, scale, causal,
                                    wl, wr, st, ws, sms);
  if (rc != FA_OK) return rc;
  // 2. dK, dV: persistent, one CTA per SM over the (b, kv head, key block) tiles
  const long long kv_tiles = (long long)B * Hkv * p.nkt;
  const unsigned kv_grid = (unsigned)(kv_tiles < sms ? kv_tiles : sms);
  if (launch_after(fab::bwd_dkdv_kernel<D, BF16, BIAS>, kv_grid, GK::SMEM_BYTES, st, tq, tdo, tk, tv, p,
                   tb, bias_mode) != cudaSuccess)
    return FA_ERR_LAUNCH;
  // 3. dQ: persistent, one CTA per SM over the (b, query head, query block) tiles
  const long long q_tiles = (long long)B * Hq * p.nqt;
  const unsigned q_grid = (unsigned)(q_tiles < sms ? q_tiles : sms);
  return launch_after(fab::bwd_dq_kernel<D, BF16, BIAS>, q_grid, GQ::SMEM_BYTES, st, tq, tdo, tk, tv, p,
                      tb, bias_mode) == cudaSuccess
             ? FA_OK
             : FA_ERR_LAUNCH;
}

}  // namespace

extern "C" {

size_t fa_bwd_workspace_size(int B, int Hq, int Nq) {
  if (B < 1 || Hq < 1 || Nq < 1) return 0;
  return 2ull * (size_t)B * Hq * nq_pad(Nq) * sizeof(float);
}

}  // extern "C"

namespace {

int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nk,
             int D, float scale, int causal, int window_left, int window_right, void* stream,
             int dtype, void* workspace, size_t workspace_bytes, const BiasArgB* bias) {
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_BAD_DTYPE;
  if (window_left < -1 || window_right < -1 || (causal && window_right > 0)) return FA_ERR_BAD_WINDOW;
  if (D != 64 && D != 128 && D != 256) return FA_ERR_UNSUPPORTED_HEAD_DIM;
  if (bias && D == 256) return FA_ERR_UNSUPPORTED_HEAD_DIM;  // no room for a bias tile
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1) return FA_ERR_BAD_SHAPE;
  if (Hq % Hkv != 0) return FA_ERR_BAD_GROUPING;
  if ((long long)B * Hq * nq_pad(Nq) >= (1ll << 31) || (long long)B * Hkv * Nk >= (1ll << 31))
    return FA_ERR_BAD_SHAPE;
  if (!std::isfinite(scale)) return FA_ERR_BAD_SCALE;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_NULL_POINTER;
  if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)o | (uintptr_t)dout |
       (uintptr_t)dq | (uintptr_t)dk | (uintptr_t)dv) & 15u)
    return FA_ERR_MISALIGNED;
  if ((uintptr_t)lse & 3u) return FA_ERR_MISALIGNED;
  if (workspace == nullptr || workspace_bytes < fa_bwd_workspace_size(B, Hq, Nq))
    return FA_ERR_BAD_WORKSPACE;
  if ((uintptr_t)workspace & 255u) return FA_ERR_MISALIGNED;
  const size_t qb = (size_t)B * Hq * Nq * D * 2, kb = (size_t)B * Hkv * Nk * D * 2;
  const size_t lb = (size_t)B * Hq * Nq * 4, wb = fa_bwd_workspace_size(B, Hq, Nq);
  const void* ins[6] = {q, k, v, o, dout, lse};
  const size_t in_b[6] = {qb, kb, kb, qb, qb, lb};
  void* outs[4] = {dq, dk, dv, workspace};
  const size_t out_b[4] = {qb, kb, kb, wb};
  for (int a = 0; a < 4; ++a) {
    for (int b = 0; b < 6; ++b)
      if (overlaps_b(outs[a], out_b[a], ins[b], in_b[b])) return FA_ERR_OVERLAP;
    for (int b = a + 1; b < 4; ++b)
      if (overlaps_b(outs[a], out_b[a], outs[b], out_b[b])) return FA_ERR_OVERLAP;
  }
  if (bias) {  // the outputs and the workspace must not overlap the bias either
    const size_t extent = 2 * static_cast<size_t>((B - 1) * bias->sb + (Hq - 1) * bias->sh +
                                                  (Nq - 1) * bias->sq + Nk);
    for (int a = 0; a < 4; ++a)
      if (overlaps_b(outs[a], out_b[a], bias->ptr, extent)) return FA_ERR_OVERLAP;
  }
  int dev = -1, major = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      major != 10 || sms < 1)
    return FA_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = dtype == FA_BF16;
#define FA_BWD_ARGS q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, scale, causal, window_left, \
                    window_right, st, workspace, sms
  if (bias) {
    if (D == 64)
      return bf ? launch_bwd<64, true, true>(FA_BWD_ARGS, bias) : launch_bwd<64, false, true>(FA_BWD_ARGS, bias);
    return bf ? launch_bwd<128, true, true>(FA_BWD_ARGS, bias) : launch_bwd<128, false, true>(FA_BWD_ARGS, bias);
  }
  if (D == 64) return bf ? launch_bwd<64, true>(FA_BWD_ARGS) : launch_bwd<64, false>(FA_BWD_ARGS);
  if (D == 256) return bf ? launch_bwd256<true>(FA_BWD_ARGS) : launch_bwd256<false>(FA_BWD_ARGS);
  return bf ? launch_bwd<128, true>(FA_BWD_ARGS) : launch_bwd<128, false>(FA_BWD_ARGS);
#undef FA_BWD_ARGS
}

}  // namespace

extern "C" {

int fa_bwd_window(const void* q, const void* k, const void* v, const void* o, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq,
                  int Nk, int D, float scale, int causal, int window_left, int window_right,
                  void* stream, int dtype, void* workspace, size_t workspace_bytes) {
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, D, scale, causal,
                  window_left, window_right, stream, dtype, workspace, workspace_bytes, nullptr);
}

int fa_bwd_bias_window(const void* q, const void* k, const void* v, const void* o,
                       const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                       int Hq, int Hkv, int Nq, int Nk, int D, float scale, int causal,
                       const void* bias, long long bias_stride_b, long long bias_stride_h,
                       long long bias_stride_q, int window_left, int window_right, void* stream,
                       int dtype, void* workspace, size_t workspace_bytes) {
  if (bias == nullptr) return FA_ERR_NULL_POINTER;
  if (bias_stride_b < 0 || bias_stride_h < 0 || bias_stride_q < 0) return FA_ERR_BAD_SHAPE;
  if ((reinterpret_cast<uintptr_t>(bias) & 15u) || (bias_stride_b & 7) || (bias_stride_h & 7) ||
      (bias_stride_q & 7))
    return FA_ERR_MISALIGNED;
  const BiasArgB a{bias, bias_stride_b, bias_stride_h, bias_stride_q};
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, D, scale, causal,
                  window_left, window_right, stream, dtype, workspace, workspace_bytes, &a);
}

int fa_bwd_bias(const void* q, const void* k, const void* v, const void* o, const void* dout,
                const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq,
                int Nk, int D, float scale, int causal, const void* bias, long long bias_stride_b,
                long long bias_stride_h, long long bias_stride_q, void* stream, int dtype,
                void* workspace, size_t workspace_bytes) {
  return fa_bwd_bias_window(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, D, scale, causal,
                            bias, bias_stride_b, bias_stride_h, bias_stride_q, -1, -1, stream,
                            dtype, workspace, workspace_bytes);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
           const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nk,
           int D, float scale, int causal, void* stream, int dtype, void* workspace,
           size_t workspace_bytes) {
  return fa_bwd_window(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, D, scale, causal, -1,
                       -1, stream, dtype, workspace, workspace_bytes);
}

// Status word of the backward kernels (read and optionally reset); used by
// fa_device_status, not part of the public interface.
__attribute__((visibility("hidden"))) int fa_bwd_device_status_internal(int reset) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, fab::g_bwd_status, sizeof(v)) != cudaSuccess) return -1;
  if (reset) {
    const unsigned int z = 0;
    const unsigned long long zz = 0;
    if (cudaMemcpyToSymbol(fab::g_bwd_status, &z, sizeof(z)) != cudaSuccess ||
        cudaMemcpyToSymbol(fab::g_bwd_site, &zz, sizeof(zz)) != cudaSuccess)
      return -1;
  }
  return static_cast<int>(v);
}

}  // extern "C"
