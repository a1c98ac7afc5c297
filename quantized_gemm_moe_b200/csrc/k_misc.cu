// Weight-only (W3A16 / W4A16) product on CUDA cores, and the token-aware
// Top-k importance statistic with its channel histogram.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "qe_internal.h"

namespace qe {
namespace {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }
__device__ __forceinline__ uint16_t f2bf(float v) {
  __nv_bfloat16 h = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t*>(&h);
}

// ------------------------------------------------------------------ weight-only
// CTA = 128 output rows x TT token positions x one K range; thread = row.
// Per 128-channel block the TT activations (bf16(x*s_inv), bucket order) are
// staged as fp32 in shared memory. Each thread decodes its row's codes, keeps
// the exact sum_k x*q per group, and folds in the group scale at the group's end.
template <int TT, int BITS>
__global__ void __launch_bounds__(128) k_wonly(const uint16_t* __restrict__ act16, const uint8_t* __restrict__ wp,
                                               const float* __restrict__ w_scale, const uint16_t* __restrict__ ucat,
                                               const float* __restrict__ su, const uint16_t* __restrict__ bcat,
                                               int R_pad, int has_adapters,
                                               const int32_t* __restrict__ perm, int T, int N, int K, int group,
                                               int kb_per_split, void* __restrict__ Y, int y_bf16,
                                               float* __restrict__ partial) {
  __shared__ __align__(16) float act[kTileK][TT];
  const int r = threadIdx.x, nt = blockIdx.x, p0 = blockIdx.y * TT, split = blockIdx.z;
  const int o = nt * kTileN + r;
  const int KB = static_cast<int>(ceil_div(K, kTileK));
  const int kb0 = split * kb_per_split, kb1 = min(KB, kb0 + kb_per_split);
  constexpr int kBlockBytes = (BITS == 4) ? kW4BlockBytes : kW3BlockBytes;
  constexpr int kRowBytes = kBlockBytes / kTileN;
  float acc[TT], part[TT];
#pragma unroll
  for (int i = 0; i < TT; ++i) acc[i] = part[i] = 0.0f;
  for (int kb = kb0; kb < kb1; ++kb) {
    __syncthreads();
    for (int i = r; i < kTileK * TT; i += blockDim.x) {
      const int kl = i / TT, tt = i % TT, k = kb * kTileK + kl, p = p0 + tt;
      act[kl][tt] = (k < K && p < T) ? bf16_bits_to_f32(act16[static_cast<size_t>(p) * K + k]) : 0.0f;
    }
    __syncthreads();
    const uint8_t* row = wp + (static_cast<size_t>(nt) * KB + kb) * kBlockBytes + r * kRowBytes;
    uint32_t wv[kRowBytes / 4];
#pragma unroll
    for (int i = 0; i < kRowBytes / 16; ++i) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(row) + i);
      wv[4 * i] = u.x; wv[4 * i + 1] = u.y; wv[4 * i + 2] = u.z; wv[4 * i + 3] = u.w;
    }
    const int gpb = kTileK / group;
#pragma unroll 1
    for (int gi = 0; gi < gpb; ++gi) {
      const int j = kb * gpb + gi;
      if (j * group >= K) break;
#pragma unroll 4
      for (int kk = 0; kk < group; ++kk) {
        const int kl = gi * group + kk;
        int qv;
        if constexpr (BITS == 4) {
          const int h = kl >> 5, i = kl & 31, hi = i >> 4, w = (i & 15) >> 2, b = i & 3;
          const uint32_t nib = (wv[4 * h + w] >> (8 * b + 4 * hi)) & 0xFu;
          qv = static_cast<int>(nib) - static_cast<int>((nib & 8u) << 1);
        } else {
          const int m = kl >> 4, pp = (kl & 15) >> 1, odd = kl & 1;
          const int hw = kl >> 5, hp = (kl & 31) >> 1;
          const uint32_t lo2 = (wv[m] >> (odd ? 16 + 2 * pp : 2 * pp)) & 3u;
          const uint32_t b2 = (wv[8 + hw] >> (odd ? 16 + hp : hp)) & 1u;
          qv = static_cast<int>(lo2 | (b2 << 2)) - 4;
        }
        const float qf = static_cast<float>(qv);
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) part[tt] = fmaf(qf, act[kl][tt], part[tt]);
      }
      const float sw = (o < N) ? __ldg(w_scale + static_cast<size_t>(j) * N + o) : 0.0f;
#pragma unroll
      for (int tt = 0; tt < TT; ++tt) {
        acc[tt] = fmaf(sw, part[tt], acc[tt]);
        part[tt] = 0.0f;
      }
    }
  }
  if (o >= N) return;
  if (has_adapters && split == 0) {
    const __half* brow = reinterpret_cast<const __half*>(bcat) + static_cast<size_t>(o) * R_pad;
    const __half* uc = reinterpret_cast<const __half*>(ucat);
    float ad[TT];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) ad[tt] = 0.0f;
    for (int c = 0; c < R_pad; ++c) {
      const float b = __half2float(brow[c]);
#pragma unroll
      for (int tt = 0; tt < TT; ++tt) {
        const int p = p0 + tt;
        if (p < T) ad[tt] = fmaf(__half2float(uc[static_cast<size_t>(p) * R_pad + c]), b, ad[tt]);
      }
    }
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
      if (p0 + tt < T) acc[tt] = fmaf(su[p0 + tt], ad[tt], acc[tt]);
  }
#pragma unroll
  for (int tt = 0; tt < TT; ++tt) {
    const int p = p0 + tt;
    if (p >= T) break;
    if (partial) {
      partial[(static_cast<size_t>(split) * T + p) * N + o] = acc[tt];
    } else {
      const size_t dst = static_cast<size_t>(perm[p]) * N + o;
      if (y_bf16) static_cast<uint16_t*>(Y)[dst] = f2bf(acc[tt]);
      else static_cast<float*>(Y)[dst] = acc[tt];
    }
  }
}

template <int TT>
cudaError_t launch_wonly_t(const uint16_t* act16, const uint8_t* wp, const float* w_scale, int w_bits,
                           const uint16_t* ucat, const float* su, const uint16_t* bcat, int R_pad, int has_adapters,
                           const int32_t* perm, int T, int N, int K, int group, void* Y, int y_bf16,
                           float* partial, int splits, cudaStream_t st) {
  const int KB = static_cast<int>(ceil_div(K, kTileK));
  const int kbps = static_cast<int>(ceil_div(KB, splits));
  dim3 grid(static_cast<unsigned>(ceil_div(N, kTileN)), static_cast<unsigned>(ceil_div(T, TT)),
            static_cast<unsigned>(splits));
  float* part = splits > 1 ? partial : nullptr;
  if (w_bits == 4)
    k_wonly<TT, 4><<<grid, 128, 0, st>>>(act16, wp, w_scale, ucat, su, bcat, R_pad, has_adapters, perm, T, N, K, group,
                                         kbps, Y, y_bf16, part);
  else
    k_wonly<TT, 3><<<grid, 128, 0, st>>>(act16, wp, w_scale, ucat, su, bcat, R_pad, has_adapters, perm, T, N, K, group,
                                         kbps, Y, y_bf16, part);
  return cudaGetLastError();
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

}  // namespace

cudaError_t launch_wonly(const uint16_t* act16, const uint8_t* w_packed, const float* w_scale, int w_bits,
                         const uint16_t* ucat, const float* su, const uint16_t* bcat, int R_pad, int has_adapters,
                         const int32_t* perm, int T, int N, int K, int group, void* Y, int y_bf16, float* partial,
                         int splits, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
#define QE_WO(TT) \
  launch_wonly_t<TT>(act16, w_packed, w_scale, w_bits, ucat, su, bcat, R_pad, has_adapters, perm, T, N, K, group, Y, \
                     y_bf16, partial, splits, st)
  if (T <= 1) return QE_WO(1);
  if (T <= 2) return QE_WO(2);
  if (T <= 4) return QE_WO(4);
  if (T <= 8) return QE_WO(8);
  return QE_WO(16);
#undef QE_WO
}

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
