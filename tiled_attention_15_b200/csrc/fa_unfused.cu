// fa_unfused.cu -- standard (unfused) attention, the comparison the pages make.
//
// The mooersco.com article ("标准 Attention 的瓶颈在哪" and the measurement table of
// "跟标准 Attention 的性能差距有多大") and section 二 of the gitcode.csdn.net article
// describe attention done in three separate steps, each going through device
// memory:
//
//   S = scale * Q K^T        (an Nq x Nk matrix per head, written out)
//   P = softmax(S) by rows   (read S back, write P out)
//   O = P V                  (read P back)
//
// This file builds that path on the GPU so the fused kernel can be compared
// with it on the same inputs: the two products are plain batched GEMMs
// (cuBLAS, fp32 accumulation; S kept in fp32 so the softmax sees unrounded
// scores), the row softmax is the kernel below (max, sum of exponentials,
// normalised P rounded to the input dtype, natural-log LSE).  S and P live in a
// caller workspace of fa_fwd_unfused_workspace_size() bytes: 6 bytes per score,
// which is what the fused kernel never writes.
#include <cublas_v2.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa.h"

namespace fau {

constexpr int kThreads = 256;

__device__ __forceinline__ float block_reduce_max(float x, float* red) {
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();  // red is reused across reductions
  if (l == 0) red[w] = x;
  __syncthreads();
  x = l < kThreads / 32 ? red[l] : -INFINITY;
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

__device__ __forceinline__ float block_reduce_sum(float x, float* red) {
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = x;
  __syncthreads();
  x = l < kThreads / 32 ? red[l] : 0.f;
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// One CTA per score row (b, h, i): m = max over the visible keys of scale * s_j,
// Z = sum exp(scale * s_j - m), P_j = exp(scale * s_j - m) / Z rounded to the
// input dtype (0 for keys the causal mask removes), LSE = m + ln Z.  For rows
// longer than the register-resident kernel below takes, the row is read three
// times; the second and third reads hit the cache.
template <bool BF16>
__global__ void __launch_bounds__(kThreads) softmax_rows_kernel(const float* __restrict__ S,
                                                                 uint16_t* __restrict__ P,
                                                                 float* __restrict__ lse, int Nq,
                                                                 int Nk, float scale, int causal) {
  __shared__ float red[kThreads / 32];
  const long long row = blockIdx.x;
  const int i = static_cast<int>(row % Nq);
  const int nvis = causal ? min(Nk, i + 1) : Nk;
  const float* s = S + row * Nk;
  uint16_t* p = P + row * Nk;
  float m = -INFINITY;
  for (int j = threadIdx.x; j < nvis; j += kThreads) m = fmaxf(m, scale * s[j]);
  m = block_reduce_max(m, red);
  float z = 0.f;
  for (int j = threadIdx.x; j < nvis; j += kThreads) z += expf(scale * s[j] - m);
  z = block_reduce_sum(z, red);
  const float inv = 1.f / z;
  for (int j = threadIdx.x; j < Nk; j += kThreads) {
    const float pj = j < nvis ? expf(scale * s[j] - m) * inv : 0.f;
    if (BF16) {
      const __nv_bfloat16 h = __float2bfloat16_rn(pj);
      p[j] = *reinterpret_cast<const uint16_t*>(&h);
    } else {
      const __half h = __float2half_rn(pj);
      p[j] = *reinterpret_cast<const uint16_t*>(&h);
    }
  }
  if (lse != nullptr && threadIdx.x == 0) lse[row] = m + logf(z);
}

// The same for rows of at most kThreads * VPT keys, with the row held in
// registers: S is read once and P written once.
template <bool BF16, int VPT>
__global__ void __launch_bounds__(kThreads) softmax_rows_reg_kernel(const float* __restrict__ S,
                                                                     uint16_t* __restrict__ P,
                                                                     float* __restrict__ lse, int Nq,
                                                                     int Nk, float scale, int causal) {
  __shared__ float red[kThreads / 32];
  const long long row = blockIdx.x;
  const int i = static_cast<int>(row % Nq);
  const int nvis = causal ? min(Nk, i + 1) : Nk;
  const float* s = S + row * Nk;
  uint16_t* p = P + row * Nk;
  float x[VPT];
  float m = -INFINITY;
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int j = threadIdx.x + k * kThreads;
    x[k] = j < nvis ? scale * s[j] : -INFINITY;
    m = fmaxf(m, x[k]);
  }
  m = block_reduce_max(m, red);
  float z = 0.f;
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    x[k] = expf(x[k] - m);  // 0 for the keys the mask removes
    z += x[k];
  }
  z = block_reduce_sum(z, red);
  const float inv = 1.f / z;
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int j = threadIdx.x + k * kThreads;
    if (j < Nk) {
      const float pj = x[k] * inv;
      if (BF16) {
        const __nv_bfloat16 h = __float2bfloat16_rn(pj);
        p[j] = *reinterpret_cast<const uint16_t*>(&h);
      } else {
        const __half h = __float2half_rn(pj);
        p[j] = *reinterpret_cast<const uint16_t*>(&h);
      }
    }
  }
  if (lse != nullptr && threadIdx.x == 0) lse[row] = m + logf(z);
}

template <bool BF16>
void launch_softmax(const float* S, uint16_t* P, float* lse, int Nq, int Nk, float scale, int causal,
                    unsigned rows, cudaStream_t st) {
  if (Nk <= kThreads * 4)
    softmax_rows_reg_kernel<BF16, 4><<<rows, kThreads, 0, st>>>(S, P, lse, Nq, Nk, scale, causal);
  else if (Nk <= kThreads * 8)
    softmax_rows_reg_kernel<BF16, 8><<<rows, kThreads, 0, st>>>(S, P, lse, Nq, Nk, scale, causal);
  else if (Nk <= kThreads * 16)
    softmax_rows_reg_kernel<BF16, 16><<<rows, kThreads, 0, st>>>(S, P, lse, Nq, Nk, scale, causal);
  else if (Nk <= kThreads * 32)
    softmax_rows_reg_kernel<BF16, 32><<<rows, kThreads, 0, st>>>(S, P, lse, Nq, Nk, scale, causal);
  else
    softmax_rows_kernel<BF16><<<rows, kThreads, 0, st>>>(S, P, lse, Nq, Nk, scale, causal);
}

}  // namespace fau

namespace {

constexpr int kMaxDevices = 64;
cublasHandle_t g_handle[kMaxDevices] = {};
std::mutex g_mu;  // one handle per device, shared: a call holds the lock while it enqueues

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

extern "C" {

size_t fa_fwd_unfused_workspace_size(int B, int Hq, int Nq, int Nk) {
  if (B < 1 || Hq < 1 || Nq < 1 || Nk < 1) return 0;
  const size_t n = static_cast<size_t>(B) * Hq * Nq * Nk;
  return up256(n * 4) + up256(n * 2);
}

int fa_fwd_unfused(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                   int Hkv, int Nq, int Nk, int D, float scale, int causal, void* stream, int dtype,
                   void* workspace, size_t workspace_bytes) {
  // ---- host checks, before any CUDA call
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_BAD_DTYPE;
  if (D != 64 && D != 128 && D != 256) return FA_ERR_UNSUPPORTED_HEAD_DIM;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1) return FA_ERR_BAD_SHAPE;
  if (Hq % Hkv != 0) return FA_ERR_BAD_GROUPING;
  if (static_cast<long long>(B) * Hq * Nq >= (1ll << 31)) return FA_ERR_BAD_SHAPE;
  if (!std::isfinite(scale)) return FA_ERR_BAD_SCALE;
  if (!q || !k || !v || !o) return FA_ERR_NULL_POINTER;
  if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)o) & 15u) return FA_ERR_MISALIGNED;
  if (lse && ((uintptr_t)lse & 3u)) return FA_ERR_MISALIGNED;
  const size_t qo_b = static_cast<size_t>(B) * Hq * Nq * D * 2, kv_b = static_cast<size_t>(B) * Hkv * Nk * D * 2;
  auto overlaps = [](const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
  };
  if (overlaps(o, qo_b, q, qo_b) || overlaps(o, qo_b, k, kv_b) || overlaps(o, qo_b, v, kv_b))
    return FA_ERR_OVERLAP;
  if (lse) {
    const size_t lb = static_cast<size_t>(B) * Hq * Nq * 4;
    if (overlaps(lse, lb, q, qo_b) || overlaps(lse, lb, k, kv_b) || overlaps(lse, lb, v, kv_b) ||
        overlaps(lse, lb, o, qo_b))
      return FA_ERR_OVERLAP;
  }
  const size_t need = fa_fwd_unfused_workspace_size(B, Hq, Nq, Nk);
  if (workspace == nullptr || workspace_bytes < need || ((uintptr_t)workspace & 255u))
    return FA_ERR_BAD_WORKSPACE;
  // ---- device
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_NO_DEVICE;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      major != 10)
    return FA_ERR_NO_DEVICE;
  const size_t n = static_cast<size_t>(B) * Hq * Nq * Nk;
  float* S = static_cast<float*>(workspace);
  uint16_t* P = reinterpret_cast<uint16_t*>(static_cast<char*>(workspace) + up256(n * 4));
  const cudaDataType_t t16 = dtype == FA_BF16 ? CUDA_R_16BF : CUDA_R_16F;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int g = Hq / Hkv;
  const long long nkd = static_cast<long long>(Nk) * D, nqd = static_cast<long long>(Nq) * D,
                  nqk = static_cast<long long>(Nq) * Nk;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_handle[dev] == nullptr && cublasCreate(&g_handle[dev]) != CUBLAS_STATUS_SUCCESS) {
    g_handle[dev] = nullptr;
    return FA_ERR_LIBRARY;
  }
  cublasHandle_t h = g_handle[dev];
  if (cublasSetStream(h, st) != CUBLAS_STATUS_SUCCESS) return FA_ERR_LIBRARY;
  const float one = 1.f, zero = 0.f;
  // Row-major X[rows][cols] is the column-major cols x rows matrix, so
  //   S[i][j] = q_i . k_j     is  S^cm (Nk x Nq) = K^cm^T (Nk x D) * Q^cm (D x Nq)
  //   O[i][d] = sum_j P[i][j] v_j[d]  is  O^cm (D x Nq) = V^cm (D x Nk) * P^cm (Nk x Nq)
  // batched over the (batch, key/value head) pairs, one call per query head of
  // a group (query head kvh * g + r reads key/value head kvh).
  for (int r = 0; r < g; ++r) {
    if (cublasGemmStridedBatchedEx(h, CUBLAS_OP_T, CUBLAS_OP_N, Nk, Nq, D, &one, k, t16, D, nkd,
                                   static_cast<const uint16_t*>(q) + r * nqd, t16, D, g * nqd,
                                   &zero, S + r * nqk, CUDA_R_32F, Nk, g * nqk, B * Hkv,
                                   CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
      return FA_ERR_LIBRARY;
  }
  const unsigned rows = static_cast<unsigned>(static_cast<long long>(B) * Hq * Nq);
  if (dtype == FA_BF16)
    fau::launch_softmax<true>(S, P, lse, Nq, Nk, scale, causal, rows, st);
  else
    fau::launch_softmax<false>(S, P, lse, Nq, Nk, scale, causal, rows, st);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  for (int r = 0; r < g; ++r) {
    if (cublasGemmStridedBatchedEx(h, CUBLAS_OP_N, CUBLAS_OP_N, D, Nq, Nk, &one, v, t16, D, nkd,
                                   P + r * nqk, t16, Nk, g * nqk, &zero,
                                   static_cast<uint16_t*>(o) + r * nqd, t16, D, g * nqd, B * Hkv,
                                   CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
      return FA_ERR_LIBRARY;
  }
  return FA_OK;
}

}  // extern "C"
