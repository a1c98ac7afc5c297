// The token-aware Top-k importance statistic with its channel histogram.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "qe_internal.h"
#include "qe_ptx.cuh"

namespace qe {
namespace {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }
__device__ __forceinline__ uint16_t f2bf(float v) {
  __nv_bfloat16 h = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t*>(&h);
}

// ------------------------------------------------------------------ Top-k importance
// One CTA per token. Scores fl32(|x|*w) are mapped to order-preserving uint32
// keys and kept in shared memory. A 4-pass MSB radix select (8-bit digits,
// per-warp histograms with warp-aggregated increments) finds the k-th largest
// key tau. An ordered collect takes every key > tau and the lowest-index keys
// == tau. A bitonic sort orders the k picks by (key desc, channel asc).
constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;

__device__ __forceinline__ uint32_t order_key(float v) {
  v = v + 0.0f;  // -0 -> +0 so that equal scores get equal keys
  const uint32_t b = __float_as_uint(v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

template <bool BF16>
__global__ void __launch_bounds__(kTopkThreads) k_topk(const void* __restrict__ X, const float* __restrict__ w,
                                                       int T, int K, int k, int32_t* __restrict__ idx_out,
                                                       int32_t* __restrict__ hist) {
  extern __shared__ uint32_t keys[];  // [K]
  __shared__ int whist[kTopkWarps][256];
  __shared__ int digits[256];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_remaining;
  __shared__ int sgt[kTopkThreads], seq[kTopkThreads];
  __shared__ unsigned long long sel[128];
  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t rowoff = static_cast<size_t>(t) * K;
  for (int k0 = tid * 8; k0 < K; k0 += kTopkThreads * 8) {
    float xv[8];
    if constexpr (BF16) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(X) + rowoff + k0));
      const uint32_t ww[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        xv[2 * i] = bf16_bits_to_f32(ww[i] & 0xFFFFu);
        xv[2 * i + 1] = bf16_bits_to_f32(ww[i] >> 16);
      }
    } else {
      const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(X) + rowoff + k0);
      const float4 a = __ldg(p), b = __ldg(p + 1);
      xv[0] = a.x; xv[1] = a.y; xv[2] = a.z; xv[3] = a.w; xv[4] = b.x; xv[5] = b.y; xv[6] = b.z; xv[7] = b.w;
    }
    const float4 wa = __ldg(reinterpret_cast<const float4*>(w + k0));
    const float4 wb = __ldg(reinterpret_cast<const float4*>(w + k0) + 1);
    const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) keys[k0 + i] = order_key(__fmul_rn(fabsf(xv[i]), wv[i]));
  }
  if (tid == 0) {
    s_prefix = 0u;
    s_mask = 0u;
    s_remaining = k;
  }
  __syncthreads();
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < kTopkWarps * 256; i += kTopkThreads) (&whist[0][0])[i] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int base = 0; base < K; base += kTopkThreads) {
      const int i = base + tid;
      const uint32_t key = (i < K) ? keys[i] : 0u;
      const bool match = (i < K) && ((key & mask) == prefix);
      const uint32_t active = __ballot_sync(0xffffffffu, match);
      if (match) {
        const int d = static_cast<int>((key >> shift) & 255u);
        const uint32_t peers = __match_any_sync(active, d);
        if (lane == __ffs(peers) - 1) whist[warp][d] += __popc(peers);
      }
    }
    __syncthreads();
    if (tid < 256) {
      int sum = 0;
#pragma unroll
      for (int w2 = 0; w2 < kTopkWarps; ++w2) sum += whist[w2][tid];
      digits[tid] = sum;
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits 255-8l .. 248-8l (descending); find where the count from the top reaches remaining
      int cnt[8];
      int lsum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[j] = digits[255 - 8 * lane - j];
        lsum += cnt[j];
      }
      int incl = lsum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      const int excl = incl - lsum;
      const int rem = s_remaining;
      const bool hit = (excl < rem) && (incl >= rem);
      const uint32_t hm = __ballot_sync(0xffffffffu, hit);
      if (lane == __ffs(hm) - 1) {
        int run = excl, d = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (run + cnt[j] >= rem) {
            d = 255 - 8 * lane - j;
            break;
          }
          run += cnt[j];
        }
        s_remaining = rem - run;
        s_prefix = prefix | (static_cast<uint32_t>(d) << shift);
        s_mask = mask | (255u << shift);
      }
    }
    __syncthreads();
  }
  const uint32_t tau = s_prefix;
  const int need_eq = s_remaining;
  const int n_gt = k - need_eq;
  // ordered collect over contiguous per-thread chunks
  const int chunk = static_cast<int>(ceil_div(K, kTopkThreads));
  const int c_lo = min(K, tid * chunk), c_hi = min(K, c_lo + chunk);
  int ngt = 0, neq = 0;
  for (int i = c_lo; i < c_hi; ++i) {
    const uint32_t key = keys[i];
    ngt += key > tau;
    neq += key == tau;
  }
  sgt[tid] = ngt;
  seq[tid] = neq;
  __syncthreads();
  // exclusive scans (Hillis-Steele in shared memory; 512 entries)
  for (int off = 1; off < kTopkThreads; off <<= 1) {
    const int a = (tid >= off) ? sgt[tid - off] : 0;
    const int b = (tid >= off) ? seq[tid - off] : 0;
    __syncthreads();
    sgt[tid] += a;
    seq[tid] += b;
    __syncthreads();
  }
  int gpos = sgt[tid] - ngt, epos = seq[tid] - neq;
  for (int i = c_lo; i < c_hi; ++i) {
    const uint32_t key = keys[i];
    const unsigned long long comp =
        (static_cast<unsigned long long>(key) << 32) | static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(i));
    if (key > tau) sel[gpos++] = comp;
    else if (key == tau) {
      if (epos < need_eq) sel[n_gt + epos] = comp;
      ++epos;
    }
  }
  int KP = 1;
  while (KP < k) KP <<= 1;
  for (int i = k + tid; i < KP; i += kTopkThreads) sel[i] = 0ull;
  __syncthreads();
  // bitonic sort, descending
  for (int size = 2; size <= KP; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < KP; i += kTopkThreads) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long a = sel[i], b = sel[j];
          if ((a < b) == desc) {
            sel[i] = b;
            sel[j] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < k; i += kTopkThreads) {
    const int c = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(sel[i] & 0xFFFFFFFFull));
    idx_out[static_cast<size_t>(t) * k + i] = c;
    if (hist) atomicAdd(hist + c, 1);
  }
}

// Self-test of the bounded waits: one thread waits on a barrier that nothing arrives on. The
// wait runs out after limit_ns, records DEVERR_SELFTEST and the kernel returns.
__global__ void k_wait_selftest(int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_for(&bar, 0, err, DEVERR_SELFTEST, limit_ns);
}

}  // namespace


cudaError_t launch_topk(const void* X, bool x_bf16, const float* w_mean, int T, int K, int k, int32_t* idx,
                        int32_t* hist, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const size_t smem = static_cast<size_t>(K) * 4;
  cudaError_t e;
  if (x_bf16) {
    e = cudaFuncSetAttribute(k_topk<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k_topk<true><<<T, kTopkThreads, smem, st>>>(X, w_mean, T, K, k, idx, hist);
  } else {
    e = cudaFuncSetAttribute(k_topk<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k_topk<false><<<T, kTopkThreads, smem, st>>>(X, w_mean, T, K, k, idx, hist);
  }
  return cudaGetLastError();
}

}  // namespace qe

namespace qe {
cudaError_t launch_wait_selftest(int* err, uint64_t limit_ns, cudaStream_t st) {
  k_wait_selftest<<<1, 32, 0, st>>>(err, limit_ns);
  return cudaGetLastError();
}
}  // namespace qe
