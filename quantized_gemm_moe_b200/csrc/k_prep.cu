// Memory-bound kernels of the QE linear layer: router + per-token absmax,
// stable token->expert bucket sort, per-token quantization, weight
// quantization / packing, adapter packing, adapter finalize, split-K reduce.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "qe_internal.h"
#include "qe_ptx.cuh"

namespace qe {

// Library-owned device state, on every device that loads this module: the error word that
// bounded waits write (here), and the fixed scratch array of qe_linear_forward_noalloc
// (QE_NOALLOC_WORKSPACE_BYTES, in qe_api.cu).
__device__ int g_device_error = 0;

void* current_context() {
  using GetCurrent = CUresult (*)(CUcontext*);
  static GetCurrent fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<GetCurrent>(nullptr);
    return reinterpret_cast<GetCurrent>(f);
  }();
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// The error word's device address, looked up once per device and context (a replaced context,
// e.g. after cudaDeviceReset, loads the module again at a new address).
int* device_error_ptr() {
  static std::mutex mu;
  static int* cached[64] = {nullptr};
  static void* ctx_of[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  void* ctx = current_context();
  if (!cached[dev] || ctx != ctx_of[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    cached[dev] = static_cast<int*>(p);
    ctx_of[dev] = current_context();
  }
  return cached[dev];
}

cudaError_t read_device_error(int* value, bool clear, cudaStream_t st) {
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(int));
  if (e != cudaSuccess) return e;
  if (clear) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
  }
  return e;
}

namespace {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v) {
  __nv_bfloat16 h = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t*>(&h);
}

// Loads 8 consecutive elements x[row][k0..k0+8) as fp32 (k0 multiple of 8, row pitch K).
template <bool BF16>
__device__ __forceinline__ void load8(const void* X, size_t row, int K, int k0, float (&v)[8]) {
  if constexpr (BF16) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(X) + row * K + k0));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
      v[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(X) + row * K + k0);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

__device__ __forceinline__ void load8f(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// One symmetric RTN code: clamp(rint(fl32(v / scale)), -qmax, qmax); zero scale -> 0.
__device__ __forceinline__ int rtn_code(float v, float scale, int qmax) {
  if (scale == 0.0f) return 0;
  float r = rintf(__fdiv_rn(v, scale));
  r = fminf(fmaxf(r, -static_cast<float>(qmax)), static_cast<float>(qmax));
  return static_cast<int>(r);
}

// Eight codes through rtn_code, packed little-endian into two words. Kept out of line: callers
// unroll their loops, and this rare path would otherwise be copied into every unrolled step.
__device__ __noinline__ uint2 rtn_code8_exact(float v0, float v1, float v2, float v3, float v4, float v5, float v6,
                                              float v7, float scale, int qmax) {
  const float v[8] = {v0, v1, v2, v3, v4, v5, v6, v7};
  uint32_t w0 = 0, w1 = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w0 |= (static_cast<uint32_t>(rtn_code(v[i], scale, qmax)) & 0xFFu) << (8 * i);
    w1 |= (static_cast<uint32_t>(rtn_code(v[4 + i], scale, qmax)) & 0xFFu) << (8 * i);
  }
  return make_uint2(w0, w1);
}

// Eight codes rtn_code(v[i], scale, qmax), packed little-endian into two words, without a division
// in the common case. inv = fl32(1/scale), the correctly rounded reciprocal. g = fl32(v*inv) differs
// from the correctly rounded quotient fl32(v/scale) by at most 3 units of 2^-24 |g|, so rint(g)
// equals rint(fl32(v/scale)) unless g lies within that distance of a half-integer; the test below
// asks for a margin of 2^-20 |g| and sends the rest through rtn_code. The fast path also needs a
// normal scale, and |g| < qmax + 0.5 so that the clamp does not bind (|v| <= absmax keeps
// |g| <= qmax (1 + 2^-22) when the scale came from this row's absmax).
// rint uses the 1.5*2^23 trick: fl32(g + 1.5*2^23) holds rint(g) (half to even) in its low bits.
__device__ __forceinline__ void rtn_code8(const float (&v)[8], float scale, float inv, bool fast, int qmax,
                                          uint32_t& w0, uint32_t& w1) {
  constexpr float kM = 12582912.0f;
  const float qmax_f = static_cast<float>(qmax) + 0.5f;
  uint32_t b[8];
  bool ok = fast;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float g = __fmul_rn(v[i], inv);
    const float t = __fadd_rn(g, kM);
    const float d = fabsf(__fsub_rn(g, __fsub_rn(t, kM)));
    ok = ok && (__fmaf_rn(fabsf(g), 9.5367431640625e-07f, d) < 0.5f) && (fabsf(g) < qmax_f);
    b[i] = __float_as_uint(t);
  }
  if (ok) {
    w0 = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    w1 = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
    return;
  }
  const uint2 w = rtn_code8_exact(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7], scale, qmax);
  w0 = w.x;
  w1 = w.y;
}
// Whether rtn_code8's fast path may be used for this scale (and its reciprocal).
__device__ __forceinline__ bool rtn_fast_ok(float scale, float inv) {
  return scale >= 1.17549435e-38f && inv < 3.0e38f;
}

// ------------------------------------------------------------------ router + absmax
// One CTA per token. logits[e] = sum_k x[k]*G[k][e] in fp32; e* = argmin (lowest e on ties);
// sa = fl32(max_k |fl32(x[k]*s_inv[k])| / qmax).
template <bool BF16, int NR>
__global__ void __launch_bounds__(256) k_route_stats(const void* __restrict__ X, const float* __restrict__ s_inv,
                                                     const uint16_t* __restrict__ G, int T, int K, int n_r,
                                                     int qmax, int32_t* __restrict__ expert,
                                                     float* __restrict__ sa, float* __restrict__ logits) {
  const int t = blockIdx.x;
  float acc[NR];
#pragma unroll
  for (int e = 0; e < NR; ++e) acc[e] = 0.0f;
  float amax = 0.0f;
  const bool want_sa = sa != nullptr;
  for (int k0 = threadIdx.x * 8; k0 < K; k0 += blockDim.x * 8) {
    float xv[8];
    load8<BF16>(X, t, K, k0, xv);
    if (want_sa) {
      float si[8];
      load8f(s_inv + k0, si);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(__fmul_rn(xv[i], si[i])));
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint16_t* g = G + static_cast<size_t>(k0 + i) * n_r;
      if constexpr (NR == 8) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(g));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[2 * j] = fmaf(xv[i], bf16_bits_to_f32(w[j] & 0xFFFFu), acc[2 * j]);
          acc[2 * j + 1] = fmaf(xv[i], bf16_bits_to_f32(w[j] >> 16), acc[2 * j + 1]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < NR; ++e)
          if (e < n_r) acc[e] = fmaf(xv[i], bf16_bits_to_f32(__ldg(g + e)), acc[e]);
      }
    }
  }
  // block reduction: warp shuffles, then one row per warp in shared memory
  __shared__ float red[8][NR + 1];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
#pragma unroll
    for (int e = 0; e < NR; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
  if (lane == 0) {
#pragma unroll
    for (int e = 0; e < NR; ++e) red[warp][e] = acc[e];
    red[warp][NR] = amax;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int nw = blockDim.x >> 5;
    float best = 0.0f;
    int beste = 0;
    float am = 0.0f;
    for (int w = 0; w < nw; ++w) am = fmaxf(am, red[w][NR]);
    for (int e = 0; e < n_r; ++e) {
      float L = 0.0f;
      for (int w = 0; w < nw; ++w) L += red[w][e];
      if (logits) logits[static_cast<size_t>(t) * n_r + e] = L;
      if (e == 0 || L < best) {
        best = L;
        beste = e;
      }
    }
    if (expert) expert[t] = beste;
    if (sa) sa[t] = __fdiv_rn(am, static_cast<float>(qmax));
  }
}

// ------------------------------------------------------------------ stable bucket sort
// Single CTA of 1024 threads. Counts per expert, then assigns positions chunk by
// chunk: warp ballots give each token its rank inside its warp, a scan over the
// 32 warps gives the warp offsets, and chunks are taken in token order, so
// the sort is stable.
__global__ void __launch_bounds__(1024) k_bucket(const int32_t* __restrict__ expert, int T, int n_r,
                                                 int32_t* __restrict__ perm, int32_t* __restrict__ pos,
                                                 int32_t* __restrict__ offsets) {
  __shared__ int cnt[kMaxRouted], base[kMaxRouted];
  __shared__ int wcnt[32][kMaxRouted], wbase[32][kMaxRouted];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < kMaxRouted) cnt[tid] = 0;
  __syncthreads();
  for (int t = tid; t < T; t += blockDim.x) atomicAdd(&cnt[expert[t]], 1);
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int e = 0; e < n_r; ++e) {
      base[e] = run;
      offsets[e] = run;
      run += cnt[e];
    }
    offsets[n_r] = run;
  }
  __syncthreads();
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int c0 = 0; c0 < T; c0 += blockDim.x) {
    const int t = c0 + tid;
    const int e = (t < T) ? expert[t] : -1;
    int rank = 0;
    for (int ee = 0; ee < n_r; ++ee) {
      const uint32_t m = __ballot_sync(0xffffffffu, e == ee);
      if (lane == 0) wcnt[warp][ee] = __popc(m);
      if (e == ee) rank = __popc(m & lt_mask);
    }
    __syncthreads();
    if (tid < n_r) {
      int run = base[tid];
      for (int w = 0; w < 32; ++w) {
        wbase[w][tid] = run;
        run += wcnt[w][tid];
      }
      base[tid] = run;
    }
    __syncthreads();
    if (t < T) {
      const int p = wbase[warp][e] + rank;
      perm[p] = t;
      if (pos) pos[t] = p;
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ per-token quantization
template <bool BF16>
__global__ void __launch_bounds__(256) k_act_quant(const void* __restrict__ X, const float* __restrict__ s_inv,
                                                   int T, int K, int qmax, const float* __restrict__ sa_tok,
                                                   const int32_t* __restrict__ pos, int8_t* __restrict__ codes,
                                                   float* __restrict__ sa_sorted, uint16_t* __restrict__ act16,
                                                   uint16_t* __restrict__ xb16, uint16_t* __restrict__ xlo16) {
  const int t = blockIdx.x;
  const size_t p = pos ? static_cast<size_t>(pos[t]) : static_cast<size_t>(t);
  const float sa = sa_tok ? sa_tok[t] : 0.0f;
  const float inv = (sa > 0.0f) ? __frcp_rn(sa) : 0.0f;
  const bool fast = rtn_fast_ok(sa, inv);
  for (int k0 = threadIdx.x * 8; k0 < K; k0 += blockDim.x * 8) {
    float xv[8], si[8];
    load8<BF16>(X, t, K, k0, xv);
    load8f(s_inv + k0, si);
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(xv[i], si[i]);
    if (codes) {
      uint32_t w0, w1;
      rtn_code8(v, sa, inv, fast, qmax, w0, w1);
      *reinterpret_cast<uint2*>(codes + p * K + k0) = make_uint2(w0, w1);
    }
    if (act16) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        w[i] = static_cast<uint32_t>(f32_to_bf16_bits(v[2 * i])) |
               (static_cast<uint32_t>(f32_to_bf16_bits(v[2 * i + 1])) << 16);
      *reinterpret_cast<uint4*>(act16 + p * K + k0) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (xb16) {
      // fp32 inputs feed the bf16 adapter GEMM as x = hi + lo, both bf16 (hi + lo carries 16 significant bits)
      uint32_t w[4], wl[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint16_t h0 = f32_to_bf16_bits(xv[2 * i]), h1 = f32_to_bf16_bits(xv[2 * i + 1]);
        w[i] = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
        const uint16_t l0 = f32_to_bf16_bits(xv[2 * i] - bf16_bits_to_f32(h0));
        const uint16_t l1 = f32_to_bf16_bits(xv[2 * i + 1] - bf16_bits_to_f32(h1));
        wl[i] = static_cast<uint32_t>(l0) | (static_cast<uint32_t>(l1) << 16);
      }
      *reinterpret_cast<uint4*>(xb16 + static_cast<size_t>(t) * K + k0) = make_uint4(w[0], w[1], w[2], w[3]);
      if (xlo16)
        *reinterpret_cast<uint4*>(xlo16 + static_cast<size_t>(t) * K + k0) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
    }
  }
  if (codes && sa_sorted && threadIdx.x == 0) sa_sorted[p] = sa;
}

// ------------------------------------------------------------------ weight quantization + packing
// One CTA per (128-row tile, 128-channel block), thread = row. Two passes over
// the block: group absmax -> scale, then codes, packed 32 codes at a time.
// With fp16 scales (s16), each group scale is rounded to fp16 (nearest even) and the codes are
// computed from the stored value; a scale beyond the fp16 range is saturated to 65504 and
// reported (device error 0x203).
template <bool BF16, int BITS>
__global__ void __launch_bounds__(128) k_quant_w(const void* __restrict__ W, const float* __restrict__ s, int N,
                                                 int K, int group, uint8_t* __restrict__ packed,
                                                 void* __restrict__ w_scale, int s16, int* err) {
  constexpr int qmax = (1 << (BITS - 1)) - 1;
  const int nt = blockIdx.x, kb = blockIdx.y, r = threadIdx.x;
  const int o = nt * kTileN + r;
  const int KB = static_cast<int>(ceil_div(K, kTileK));
  const int kbase = kb * kTileK;
  const bool row_ok = o < N;
  auto wval = [&](int k) -> float {
    if (!row_ok || k >= K) return 0.0f;
    const size_t i = static_cast<size_t>(o) * K + k;
    const float w = BF16 ? bf16_bits_to_f32(static_cast<const uint16_t*>(W)[i]) : static_cast<const float*>(W)[i];
    return __fmul_rn(w, s[k]);
  };
  float sc[2] = {0.0f, 0.0f};
  const int gpb = kTileK / group;  // groups per block: 1 (g=128) or 2 (g=64)
  for (int gi = 0; gi < gpb; ++gi) {
    const int k0 = kbase + gi * group;
    if (k0 >= K) break;
    float amax = 0.0f;
    for (int k = k0; k < k0 + group; ++k) amax = fmaxf(amax, fabsf(wval(k)));
    sc[gi] = __fdiv_rn(amax, static_cast<float>(qmax));
    const size_t at = static_cast<size_t>(k0 / group) * N + o;
    if (s16) {
      __half h = __float2half_rn(sc[gi]);
      if (__hisinf(h)) {
        h = __ushort_as_half(static_cast<unsigned short>(0x7BFFu));  // 65504
        if (row_ok) record_error(err, 0x203);
      }
      sc[gi] = __half2float(h);
      if (row_ok) static_cast<__half*>(w_scale)[at] = h;
    } else if (row_ok) {
      static_cast<float*>(w_scale)[at] = sc[gi];
    }
  }
  const size_t block = static_cast<size_t>(nt) * KB + kb;
  for (int h = 0; h < 4; ++h) {  // 32 codes at a time
    int q[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int kl = 32 * h + i;
      const int k = kbase + kl;
      q[i] = (k < K) ? rtn_code(wval(k), sc[kl / group], qmax) : 0;
    }
    if constexpr (BITS == 4) {
      uint32_t wd[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t x = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const uint32_t lo = static_cast<uint32_t>(q[4 * w + b]) & 0xFu;
          const uint32_t hi = static_cast<uint32_t>(q[16 + 4 * w + b]) & 0xFu;
          x |= (lo | (hi << 4)) << (8 * b);
        }
        wd[w] = x;
      }
      *reinterpret_cast<uint4*>(packed + block * kW4BlockBytes + r * 64 + h * 16) =
          make_uint4(wd[0], wd[1], wd[2], wd[3]);
    } else {
      uint32_t two[2] = {0u, 0u}, one = 0u;
#pragma unroll
      for (int mm = 0; mm < 2; ++mm)
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const uint32_t u0 = static_cast<uint32_t>(q[16 * mm + 2 * p] + 4);
          const uint32_t u1 = static_cast<uint32_t>(q[16 * mm + 2 * p + 1] + 4);
          two[mm] |= ((u0 & 3u) << (2 * p)) | ((u1 & 3u) << (16 + 2 * p));
        }
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        const uint32_t u0 = static_cast<uint32_t>(q[2 * p] + 4);
        const uint32_t u1 = static_cast<uint32_t>(q[2 * p + 1] + 4);
        one |= ((u0 >> 2) & 1u) << p;
        one |= ((u1 >> 2) & 1u) << (16 + p);
      }
      uint8_t* row = packed + block * kW3BlockBytes + r * 48;
      *reinterpret_cast<uint2*>(row + 8 * h) = make_uint2(two[0], two[1]);
      *reinterpret_cast<uint32_t*>(row + 32 + 4 * h) = one;
    }
  }
}

// w_mean[k] = (sum_o |W[o][k]| in fp64) / N rounded once; w_colmax[k] = max_o |W[o][k]|.
template <bool BF16>
__global__ void __launch_bounds__(64) k_colstats(const void* __restrict__ W, int N, int K,
                                                 float* __restrict__ w_mean, float* __restrict__ w_colmax) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  double sum = 0.0;
  float mx = 0.0f;
  for (int o = 0; o < N; ++o) {
    const size_t i = static_cast<size_t>(o) * K + k;
    const float w = BF16 ? bf16_bits_to_f32(__ldg(static_cast<const uint16_t*>(W) + i))
                         : __ldg(static_cast<const float*>(W) + i);
    const float a = fabsf(w);
    sum += static_cast<double>(a);
    mx = fmaxf(mx, a);
  }
  if (w_mean) w_mean[k] = static_cast<float>(sum / static_cast<double>(N));
  if (w_colmax) w_colmax[k] = mx;
}

// The stored smoothing factor of the activations: s_inv[k] = fl32(1/s[k]), one correctly rounded
// IEEE division per channel (the activations are divided by s, Method, "Shared Expert").
__global__ void k_recip(const float* __restrict__ s, int K, float* __restrict__ s_inv) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k < K) s_inv[k] = __fdiv_rn(1.0f, s[k]);
}

// Inverse of the packing above (diagnostics).
template <int BITS>
__global__ void __launch_bounds__(128) k_unpack_w(const uint8_t* __restrict__ packed, int N, int K,
                                                  int8_t* __restrict__ codes) {
  const int nt = blockIdx.x, kb = blockIdx.y, r = threadIdx.x;
  const int o = nt * kTileN + r;
  if (o >= N) return;
  const int KB = static_cast<int>(ceil_div(K, kTileK));
  const size_t block = static_cast<size_t>(nt) * KB + kb;
  for (int kl = 0; kl < kTileK; ++kl) {
    const int k = kb * kTileK + kl;
    if (k >= K) break;
    int q;
    if constexpr (BITS == 4) {
      const int h = kl / 32, i = kl % 32;
      const int hi = i / 16, w = (i % 16) / 4, b = i % 4;
      const uint8_t byte = packed[block * kW4BlockBytes + r * 64 + h * 16 + 4 * w + b];
      const int nib = hi ? (byte >> 4) : (byte & 0xF);
      q = (nib & 8) ? nib - 16 : nib;
    } else {
      const uint8_t* row = packed + block * kW3BlockBytes + r * 48;
      const int m = kl / 16, p = (kl % 16) / 2, odd = kl & 1;
      const uint32_t two = *reinterpret_cast<const uint32_t*>(row + 4 * m);
      const int hword = kl / 32, hp = (kl % 32) / 2;
      const uint32_t one = *reinterpret_cast<const uint32_t*>(row + 32 + 4 * hword);
      const uint32_t lo2 = (two >> (odd ? 16 + 2 * p : 2 * p)) & 3u;
      const uint32_t b2 = (one >> (odd ? 16 + hp : hp)) & 1u;
      q = static_cast<int>(lo2 | (b2 << 2)) - 4;
    }
    codes[static_cast<size_t>(o) * K + k] = static_cast<int8_t>(q);
  }
}

// Adapter packing: A_catT [R_pad][K], B_catT [N][R_pad], G copy [K][n_r], all bf16.
// A_catT [R_tot][K] bf16 (down-projections, then the router G in rows R_pad..R_pad+N_r) and
// B_catT [N][R_pad] fp16 (up-projections). The up-projections are fp16 because the epilogue
// MMA multiplies them with the fp16 U_cat; a bf16 value beyond the fp16 range is saturated
// and reported (device error 0x201).
// Cluster-sparse routed experts (kc > 0): A_r is [n_r][kc][r_r] over the channels ch[n_r][kc];
// they are copied to rch/rar (a channel outside [0, K) becomes channel 0 with zero weights and is
// reported as device error 0x202), and A_catT holds no routed rows.
__global__ void k_pack_adapters(int K, int N, int r_s, int n_r, int r_r, int R_a, int R_pad, int R_tot, int R_rt,
                                int kc, const uint16_t* __restrict__ A_s, const uint16_t* __restrict__ B_s,
                                const uint16_t* __restrict__ A_r, const uint16_t* __restrict__ B_r,
                                const uint16_t* __restrict__ G, const int32_t* __restrict__ ch,
                                uint16_t* __restrict__ acat, uint16_t* __restrict__ bcat,
                                int32_t* __restrict__ rch, uint16_t* __restrict__ rar, int* __restrict__ err) {
  const size_t n1 = static_cast<size_t>(R_tot) * K, n2 = static_cast<size_t>(N) * R_pad;
  const size_t n3 = static_cast<size_t>(n_r) * kc, n4 = n3 * (kc ? r_r : 0);
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n1 + n2 + n3 + n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    if (i >= n1 + n2) {
      const size_t ii = i - n1 - n2;
      if (ii < n3) {
        const int c = ch[ii];
        const bool ok = c >= 0 && c < K;
        if (!ok && err) atomicCAS(err, 0, 0x202);
        rch[ii] = ok ? c : 0;
      } else {
        const size_t jj = ii - n3;  // (e * kc + i) * r_r + j
        const int c = ch[jj / r_r];
        rar[jj] = (c >= 0 && c < K) ? A_r[jj] : 0;
      }
      continue;
    }
    if (i < n1) {
      const int c = static_cast<int>(i / K), k = static_cast<int>(i % K);
      uint16_t v = 0;
      if (c < r_s) v = A_s[static_cast<size_t>(k) * r_s + c];
      else if (kc == 0 && c < R_a) {
        const int e = (c - r_s) / r_r, j = (c - r_s) % r_r;
        v = A_r[(static_cast<size_t>(e) * K + k) * r_r + j];
      } else if (c >= R_rt && c < R_rt + n_r) {
        v = G[static_cast<size_t>(k) * n_r + (c - R_rt)];
      }
      acat[i] = v;
    } else {
      const size_t ii = i - n1;
      const int o = static_cast<int>(ii / R_pad), c = static_cast<int>(ii % R_pad);
      uint16_t v = 0;
      if (c < r_s) v = B_s[static_cast<size_t>(c) * N + o];
      else if (c < R_a) {
        const int e = (c - r_s) / r_r, j = (c - r_s) % r_r;
        v = B_r[(static_cast<size_t>(e) * r_r + j) * N + o];
      }
      float f = bf16_bits_to_f32(v);
      if (fabsf(f) > 65504.0f) {
        f = copysignf(65504.0f, f);
        if (err) atomicCAS(err, 0, 0x201);
      }
      __half hv = __float2half_rn(f);
      bcat[ii] = *reinterpret_cast<uint16_t*>(&hv);
    }
  }
}

// fp32 inputs: hi = bf16(x), lo = bf16(x - hi) in token order, and amax[t] = max_k |fl32(x*s_inv)|.
// One warp per token.
__global__ void k_split_f32(const float* __restrict__ X, const float* __restrict__ s_inv, int T, int K,
                            uint16_t* __restrict__ xhi, uint16_t* __restrict__ xlo, float* __restrict__ amax) {
  const int t = static_cast<int>((blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  float mx = 0.0f;
  for (int k0 = lane * 8; k0 < K; k0 += 256) {
    float xv[8], si[8];
    load8<false>(X, t, K, k0, xv);
    load8f(s_inv + k0, si);
    uint32_t wh[4], wl[4];
#pragma unroll
    for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(__fmul_rn(xv[i], si[i])));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint16_t h0 = f32_to_bf16_bits(xv[2 * i]), h1 = f32_to_bf16_bits(xv[2 * i + 1]);
      wh[i] = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
      const uint16_t l0 = f32_to_bf16_bits(xv[2 * i] - bf16_bits_to_f32(h0));
      const uint16_t l1 = f32_to_bf16_bits(xv[2 * i + 1] - bf16_bits_to_f32(h1));
      wl[i] = static_cast<uint32_t>(l0) | (static_cast<uint32_t>(l1) << 16);
    }
    *reinterpret_cast<uint4*>(xhi + static_cast<size_t>(t) * K + k0) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
    *reinterpret_cast<uint4*>(xlo + static_cast<size_t>(t) * K + k0) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) amax[t] = mx;
}

// Sum over the GEMM's partial slots of one value, p[s * slot_stride] for s < nslots, in slot
// order, with eight loads in flight. The padding terms are +0.0f and leave the sum unchanged.
__device__ __forceinline__ float slot_sum(const float* __restrict__ p, size_t slot_stride, int nslots) {
  float acc = 0.0f;
  for (int s = 0; s < nslots; s += 8) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = (s + i < nslots) ? __ldg(p + static_cast<size_t>(s + i) * slot_stride) : 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc += v[i];
  }
  return acc;
}

// Sum of slots j, j + g, j + 2g, ... of one column, in that order, eight loads in flight.
__device__ __forceinline__ float slot_sum_strided(const float* __restrict__ p, size_t slot_stride, int nslots, int j,
                                                  int g) {
  float acc = 0.0f;
  for (int s0 = j; s0 < nslots; s0 += 8 * g) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int s = s0 + i * g;
      v[i] = (s < nslots) ? __ldg(p + static_cast<size_t>(s) * slot_stride) : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) acc += v[i];
  }
  return acc;
}

// Grid-wide barrier for a cooperative launch: every CTA is resident, so each waits until all
// have arrived. *ctr must be 0 when the kernel starts. The wait gives up after about two
// seconds of clock cycles, records an error and returns false.
__device__ bool grid_barrier(unsigned* ctr, int* err) {
  __shared__ int ok_s;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, 1u);
    int ok = 1;
    const long long t0 = clock64();
    while (true) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
      if (v >= gridDim.x) break;
      if (clock64() - t0 > 4000000000ll) {
        record_error(err, DEVERR_GRID_BARRIER);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    ok_s = ok;
  }
  __syncthreads();
  return ok_s != 0;
}

// Routing, stable bucket sort and activation quantization of one layer call, in one cooperative
// launch. CTA c owns the contiguous token range [c*chunk, (c+1)*chunk), one warp per token.
//  route:  logits = sum of the U GEMM partial slots in columns [R_pad, R_pad+N_r); expert[t] =
//          argmin (lowest index on exact ties); sa_tok[t] = fl32(max_k |fl32(x*s_inv)| / qmax), the
//          absmax read from X (bf16 inputs) or amax[t] (fp32 inputs); per-CTA expert counts.
//  (grid barrier)
//  sort:   each CTA adds the counts of all experts before e and of all earlier CTAs for e, then
//          ranks its own tokens in token order (warp ballots), so the sort is stable:
//          perm[p] = t, pos[t] = p, offsets[e].
//  quant:  at row p = pos[t]: the activation codes (or bf16(x*s_inv) for weight-only layers),
//          sa_sorted[p], and U_cat[p] = fp16((sum of U slots, routed columns of the other experts
//          zeroed) / su[p]), su[p] a power of two that puts the row's largest |U| in [2^13, 2^14).
struct RouteQuantArgs {
  const float* partial;
  int nslots, R_tot, R_pad, R_rt, n_r, r_s, r_r, R_a;
  int kc;               // cluster-sparse routed experts: channels per expert (0: dense)
  const int32_t* rch;   // [n_r][kc]
  const uint16_t* rar;  // bf16 [n_r][kc][r_r]
  const void* X;
  const float* s_inv;
  const float* amax;
  int T, K, qmax, chunk;
  int do_route, do_quant;
  int32_t* expert;
  float* sa_tok;
  int32_t* perm;
  int32_t* pos;
  int32_t* offsets;
  int32_t* counts;  // [gridDim.x][kMaxRouted]
  unsigned* barrier;
  int8_t* codes;
  uint16_t* act16;
  float* sa_sorted;
  uint16_t* ucat;
  float* su_sorted;
  unsigned* zero_words;
  int n_zero_words;
  int* err;
};

constexpr int kRQThreads = 512;
// Row loads in flight per lane: 8 x 16 B of a bf16 row, 4 x 32 B of an fp32 row.
template <bool BF16>
struct RowBatch {
  static constexpr int kIters = BF16 ? 8 : 4;
};

// Raw bytes of x[t][k0 .. k0+8) for the batch's iterations (k0 = lane*8 + 256*j), loaded first so
// that every load of the batch is in flight before any is used.
template <bool BF16>
struct RowRaw {
  uint4 v[RowBatch<BF16>::kIters][BF16 ? 1 : 2];
};
template <bool BF16>
__device__ __forceinline__ void row_load(const void* X, size_t t, int K, int k0, RowRaw<BF16>& r) {
#pragma unroll
  for (int j = 0; j < RowBatch<BF16>::kIters; ++j) {
    const int k = k0 + 256 * j;
    if (k < K) {
      if constexpr (BF16) {
        r.v[j][0] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(X) + t * K + k));
      } else {
        const uint4* q = reinterpret_cast<const uint4*>(static_cast<const float*>(X) + t * K + k);
        r.v[j][0] = __ldg(q);
        r.v[j][1] = __ldg(q + 1);
      }
    }
  }
}
// v[i] = fl32(x[k+i] * s_inv[k+i]) for iteration j of the batch (s_inv from shared memory).
template <bool BF16>
__device__ __forceinline__ void row_scaled(const RowRaw<BF16>& r, int j, const float* s_inv_s, int k, float (&v)[8]) {
  float xv[8];
  if constexpr (BF16) {
    const uint32_t w[4] = {r.v[j][0].x, r.v[j][0].y, r.v[j][0].z, r.v[j][0].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xv[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
      xv[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
  } else {
    const uint4 a0 = r.v[j][0], a1 = r.v[j][1];
    xv[0] = __uint_as_float(a0.x); xv[1] = __uint_as_float(a0.y); xv[2] = __uint_as_float(a0.z); xv[3] = __uint_as_float(a0.w);
    xv[4] = __uint_as_float(a1.x); xv[5] = __uint_as_float(a1.y); xv[6] = __uint_as_float(a1.z); xv[7] = __uint_as_float(a1.w);
  }
  const float4 s0 = *reinterpret_cast<const float4*>(s_inv_s + k);
  const float4 s1 = *reinterpret_cast<const float4*>(s_inv_s + k + 4);
  const float si[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(xv[i], si[i]);
}

// Dynamic shared memory of k_route_quant: s_inv (K floats), one adapter row per warp (R_pad floats
// each), then the range's expert ids, bucket positions and absmax bits (chunk ints each).
size_t route_quant_smem(int K, int chunk, int R_pad) {
  return size_t(K) * 4 + size_t(kRQThreads / 32) * R_pad * 4 + size_t(chunk) * 12;
}

template <bool BF16>
__global__ void __launch_bounds__(kRQThreads) k_route_quant(const RouteQuantArgs a) {
  constexpr int kWarps = kRQThreads / 32;
  constexpr int kB = RowBatch<BF16>::kIters;
  __shared__ int wcnt[kWarps][kMaxRouted], wbase[kWarps][kMaxRouted];
  __shared__ int tot_s[kMaxRouted], before_s[kMaxRouted], run_s[kMaxRouted];
  __shared__ float lpart_s[kRQThreads];  // router-logit partials of the token groups ([group][g][n_r])
  __shared__ float gmx_s[kWarps];        // per-warp maxima of a group's adapter row
  extern __shared__ float4 rq_dyn[];
  float* s_inv_s = reinterpret_cast<float*>(rq_dyn);
  float* u_w = s_inv_s + a.K;
  int* e_s = reinterpret_cast<int*>(u_w + kWarps * a.R_pad);
  int* pos_s = e_s + a.chunk;
  int* mx_s = pos_s + a.chunk;  // per-token absmax as int bits (non-negative floats order as ints)
  const size_t slot_stride = static_cast<size_t>(a.T) * a.R_tot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = min(a.T, static_cast<int>(blockIdx.x) * a.chunk), t1 = min(a.T, t0 + a.chunk);
  const int n_r = a.n_r;
  // With fewer tokens than warps, wpt warps share a token's row (wpt a power of two).
  int wpt = 1;
  while (wpt * 2 * a.chunk <= kWarps) wpt *= 2;
  const int sub = warp % wpt, slot = warp / wpt, nslot_w = kWarps / wpt;
  // A token's wpt warps meet at named barrier 1 + slot when they share its slot sums (wpt >= 2).
  const int gthr = wpt * 32, gtid = sub * 32 + lane;
  auto group_sync = [&]() { asm volatile("bar.sync %0, %1;" ::"r"(1 + slot), "r"(gthr) : "memory"); };
  for (int i = threadIdx.x; i < a.K / 4; i += kRQThreads)
    reinterpret_cast<float4*>(s_inv_s)[i] = __ldg(reinterpret_cast<const float4*>(a.s_inv) + i);
  for (int i = threadIdx.x; i < t1 - t0; i += kRQThreads) mx_s[i] = 0;
  // the decode product's tile counters start at zero (the product runs after this launch)
  for (int i = blockIdx.x * kRQThreads + threadIdx.x; i < a.n_zero_words; i += gridDim.x * kRQThreads)
    a.zero_words[i] = 0u;
  __syncthreads();

  if (a.do_route) {
    // ---- per token: logits, argmin (the token's first warp), absmax (all of its warps)
    for (int t = t0 + slot; t < t1; t += nslot_w) {
      // with several warps per token, they split each logit's slot sum: thread (j, e) adds slots
      // j, j + g, ... of column e, and the token's first warp adds the g partials in order
      const int lg = gthr / n_r;
      float* lp = lpart_s + slot * gthr;
      if (wpt > 1) {
        if (gtid < lg * n_r)
          lp[gtid] = slot_sum_strided(a.partial + static_cast<size_t>(t) * a.R_tot + a.R_rt + gtid % n_r, slot_stride,
                                      a.nslots, gtid / n_r, lg);
        group_sync();
      }
      if (sub == 0) {
        float L = 0.0f;
        if (lane < n_r) {
          if (wpt > 1) {
            for (int j = 0; j < lg; ++j) L += lp[j * n_r + lane];
          } else {
            L = slot_sum(a.partial + static_cast<size_t>(t) * a.R_tot + a.R_rt + lane, slot_stride, a.nslots);
          }
        }
        float best = (lane < n_r) ? L : INFINITY;
        int bi = (lane < n_r) ? lane : 0x7fffffff;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, best, off);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
          if (ov < best || (ov == best && oi < bi)) {
            best = ov;
            bi = oi;
          }
        }
        if (lane == 0) {
          a.expert[t] = bi;
          e_s[t - t0] = bi;
        }
      }
      if (a.sa_tok && BF16) {
        float mx = 0.0f;
        for (int k0 = (sub * 32 + lane) * 8; k0 < a.K; k0 += 256 * wpt * kB) {
          RowRaw<true> r;
#pragma unroll
          for (int j = 0; j < kB; ++j) {
            const int k = k0 + 256 * wpt * j;
            if (k < a.K)
              r.v[j][0] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.X) +
                                                                static_cast<size_t>(t) * a.K + k));
          }
#pragma unroll
          for (int j = 0; j < kB; ++j) {
            const int k = k0 + 256 * wpt * j;
            if (k < a.K) {
              float v[8];
              row_scaled<true>(r, j, s_inv_s, k, v);
#pragma unroll
              for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(v[i]));
            }
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) atomicMax(&mx_s[t - t0], __float_as_int(mx));
      }
    }
    __syncthreads();
    if (a.sa_tok) {
      for (int i = threadIdx.x; i < t1 - t0; i += kRQThreads) {
        const float mx = BF16 ? __int_as_float(mx_s[i]) : a.amax[t0 + i];
        const float sa = __fdiv_rn(mx, static_cast<float>(a.qmax));
        a.sa_tok[t0 + i] = sa;
        mx_s[i] = __float_as_int(sa);  // the quantization below reads it from here
      }
    }
    // ---- this CTA's count per expert
    if (warp < n_r) {
      int c = 0;
      for (int i = lane; i < t1 - t0; i += 32) c += (e_s[i] == warp) ? 1 : 0;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
      if (lane == 0) a.counts[blockIdx.x * kMaxRouted + warp] = c;
    }
    // ---- stable ranks inside this CTA's range (they need no other CTA), kRQThreads tokens at a
    //      time: pos_s holds each token's rank among this CTA's tokens of its expert
    if (threadIdx.x < n_r) run_s[threadIdx.x] = 0;
    __syncthreads();
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int c0 = t0; c0 < t1; c0 += kRQThreads) {
      const int t = c0 + static_cast<int>(threadIdx.x);
      const int e = (t < t1) ? e_s[t - t0] : -1;
      int rank = 0;
      for (int ee = 0; ee < n_r; ++ee) {
        const uint32_t m = __ballot_sync(0xffffffffu, e == ee);
        if (lane == 0) wcnt[warp][ee] = __popc(m);
        if (e == ee) rank = __popc(m & lt_mask);
      }
      __syncthreads();
      if (threadIdx.x < n_r) {
        int run = run_s[threadIdx.x];
        for (int w = 0; w < kWarps; ++w) {
          wbase[w][threadIdx.x] = run;
          run += wcnt[w][threadIdx.x];
        }
        run_s[threadIdx.x] = run;
      }
      __syncthreads();
      if (t < t1) pos_s[t - t0] = wbase[warp][e] + rank;
      __syncthreads();
    }
    if (!grid_barrier(a.barrier, a.err)) return;
    // ---- bucket offsets: experts before e, plus earlier CTAs' tokens of e
    if (warp < n_r) {
      int tot = 0, before = 0;
#pragma unroll 8
      for (int c = lane; c < static_cast<int>(gridDim.x); c += 32) {
        const int v = __ldcg(a.counts + c * kMaxRouted + warp);
        tot += v;
        before += (c < static_cast<int>(blockIdx.x)) ? v : 0;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        tot += __shfl_xor_sync(0xffffffffu, tot, off);
        before += __shfl_xor_sync(0xffffffffu, before, off);
      }
      if (lane == 0) {
        tot_s[warp] = tot;
        before_s[warp] = before;
      }
    }
    __syncthreads();
    if (threadIdx.x < n_r) {
      int start = 0;
      for (int e = 0; e < static_cast<int>(threadIdx.x); ++e) start += tot_s[e];
      run_s[threadIdx.x] = start + before_s[threadIdx.x];
      if (blockIdx.x == 0) {
        a.offsets[threadIdx.x] = start;
        if (threadIdx.x == n_r - 1) a.offsets[n_r] = start + tot_s[threadIdx.x];
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < t1 - t0; i += kRQThreads) {
      const int p = run_s[e_s[i]] + pos_s[i];
      a.perm[p] = t0 + i;
      a.pos[t0 + i] = p;
      pos_s[i] = p;
    }
    __syncthreads();
  } else if (a.do_quant) {
    for (int i = threadIdx.x; i < t1 - t0; i += kRQThreads) {
      pos_s[i] = a.pos[t0 + i];
      e_s[i] = a.expert[t0 + i];
    }
    __syncthreads();
  }
  if (!a.do_quant) return;
  // ---- per token, in bucket order (the token's warps share the row; its first warp writes the rest)
  for (int t = t0 + slot; t < t1; t += nslot_w) {
    const size_t p = static_cast<size_t>(pos_s[t - t0]);
    const float sa = a.codes ? (a.do_route ? __int_as_float(mx_s[t - t0]) : a.sa_tok[t]) : 0.0f;
    const float inv = (sa > 0.0f) ? __frcp_rn(sa) : 0.0f;
    const bool fast = rtn_fast_ok(sa, inv);
    for (int k0 = (sub * 32 + lane) * 8; k0 < a.K; k0 += 256 * wpt * kB) {
      RowRaw<BF16> r;
#pragma unroll
      for (int j = 0; j < kB; ++j) {
        const int k = k0 + 256 * wpt * j;
        if (k < a.K) {
          if constexpr (BF16) {
            r.v[j][0] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.X) +
                                                              static_cast<size_t>(t) * a.K + k));
          } else {
            const uint4* q = reinterpret_cast<const uint4*>(static_cast<const float*>(a.X) + static_cast<size_t>(t) * a.K + k);
            r.v[j][0] = __ldg(q);
            r.v[j][1] = __ldg(q + 1);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < kB; ++j) {
        const int k = k0 + 256 * wpt * j;
        if (k >= a.K) break;
        float v[8];
        row_scaled<BF16>(r, j, s_inv_s, k, v);
        if (a.codes) {
          uint32_t w0, w1;
          rtn_code8(v, sa, inv, fast, a.qmax, w0, w1);
          *reinterpret_cast<uint2*>(a.codes + p * a.K + k) = make_uint2(w0, w1);
        } else {
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            w[i] = static_cast<uint32_t>(f32_to_bf16_bits(v[2 * i])) |
                   (static_cast<uint32_t>(f32_to_bf16_bits(v[2 * i + 1])) << 16);
          *reinterpret_cast<uint4*>(a.act16 + p * a.K + k) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    if (wpt > 1 && a.kc == 0 && a.R_pad > 0) {
      // the token's wpt warps build its adapter row together: thread (j, c) adds slots j, j + g,
      // ... of column c into a partial row, then column c's g partials are added in order
      if (sub == 0 && a.codes && lane == 0) a.sa_sorted[p] = sa;
      const int e = e_s[t - t0];
      const int g = max(1, gthr / a.R_pad);
      float* part = u_w + static_cast<size_t>(slot) * wpt * a.R_pad;  // the group's wpt rows: [g][R_pad]
      float* row = part + static_cast<size_t>(g) * a.R_pad;           // then the summed row (g + 1 <= wpt)
      const float* prow = a.partial + static_cast<size_t>(t) * a.R_tot;
      for (int idx = gtid; idx < g * a.R_pad; idx += gthr) {
        const int c = idx % a.R_pad, j = idx / a.R_pad;
        float v = 0.0f;
        if (c < a.R_a && (c < a.r_s || (c - a.r_s) / a.r_r == e)) v = slot_sum_strided(prow + c, slot_stride, a.nslots, j, g);
        part[idx] = v;
      }
      group_sync();
      float mx = 0.0f;
      for (int c = gtid; c < a.R_pad; c += gthr) {
        float v = 0.0f;
        for (int j = 0; j < g; ++j) v += part[j * a.R_pad + c];
        row[c] = v;
        mx = fmaxf(mx, fabsf(v));
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      if (lane == 0) gmx_s[warp] = mx;
      group_sync();
      mx = 0.0f;
      for (int w = 0; w < wpt; ++w) mx = fmaxf(mx, gmx_s[slot * wpt + w]);
      float su = 1.0f;
      if (mx > 0.0f) {
        int ex;
        frexpf(mx, &ex);  // mx = m * 2^ex, m in [0.5, 1)
        su = ldexpf(1.0f, ex - 14);
      }
      const float inv_su = 1.0f / su;  // exact: su is a power of two
      for (int c = gtid; c < a.R_pad; c += gthr) {
        __half h = __float2half_rn(row[c] * inv_su);
        a.ucat[p * a.R_pad + c] = *reinterpret_cast<uint16_t*>(&h);
      }
      if (gtid == 0) a.su_sorted[p] = su;
      group_sync();  // the rows are free for the group's next token
      continue;
    }
    if (sub != 0) continue;
    if (a.codes && lane == 0) a.sa_sorted[p] = sa;
    if (a.R_pad > 0) {
      // the token's adapter row: shared columns and its own expert's routed columns are the
      // sums of the U slots; the others stay zero
      const int e = e_s[t - t0];
      float* uw = u_w + warp * a.R_pad;
      const float* prow = a.partial + static_cast<size_t>(t) * a.R_tot;
      float mx = 0.0f;
      for (int c = lane; c < a.R_pad; c += 32) {
        float v = 0.0f;
        if (c < a.R_a && (c < a.r_s || (a.kc == 0 && (c - a.r_s) / a.r_r == e)))
          v = slot_sum(prow + c, slot_stride, a.nslots);
        uw[c] = v;
        mx = fmaxf(mx, fabsf(v));
      }
      if (a.kc > 0) {
        // cluster-sparse expert: its routed columns gather the expert's channels of the raw row
        __syncwarp();
        const int32_t* chs = a.rch + static_cast<size_t>(e) * a.kc;
        const uint16_t* ar = a.rar + static_cast<size_t>(e) * a.kc * a.r_r;
        for (int j0 = 0; j0 < a.r_r; j0 += 8) {
          float acc[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) acc[jj] = 0.0f;
          for (int i = lane; i < a.kc; i += 32) {
            const int c = chs[i];
            const float x = BF16 ? bf16_bits_to_f32(static_cast<const uint16_t*>(a.X)[static_cast<size_t>(t) * a.K + c])
                                 : static_cast<const float*>(a.X)[static_cast<size_t>(t) * a.K + c];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
              if (j0 + jj < a.r_r) acc[jj] = fmaf(x, bf16_bits_to_f32(ar[static_cast<size_t>(i) * a.r_r + j0 + jj]), acc[jj]);
          }
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc[jj] += __shfl_xor_sync(0xffffffffu, acc[jj], off);
          }
          if (lane < 8 && j0 + lane < a.r_r) {
            float v = acc[0];
#pragma unroll
            for (int jj = 1; jj < 8; ++jj)
              if (lane == jj) v = acc[jj];
            uw[a.r_s + e * a.r_r + j0 + lane] = v;
            mx = fmaxf(mx, fabsf(v));
          }
        }
        __syncwarp();
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      float su = 1.0f;
      if (mx > 0.0f) {
        int ex;
        frexpf(mx, &ex);  // mx = m * 2^ex, m in [0.5, 1)
        su = ldexpf(1.0f, ex - 14);
      }
      const float inv_su = 1.0f / su;  // exact: su is a power of two
      for (int c = lane; c < a.R_pad; c += 32) {
        __half h = __float2half_rn(uw[c] * inv_su);
        a.ucat[p * a.R_pad + c] = *reinterpret_cast<uint16_t*>(&h);
      }
      if (lane == 0) a.su_sorted[p] = su;
    }
  }
}

// Y[perm[p]][o] = sum_s partial[s][p][o] (fixed order).
__global__ void k_splitk_reduce(const float* __restrict__ partial, int splits, const int32_t* __restrict__ perm,
                                int T, int N, void* __restrict__ Y, int y_bf16) {
  const size_t idx = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (idx >= static_cast<size_t>(T) * N) return;
  const int p = static_cast<int>(idx / N), o = static_cast<int>(idx % N);
  float v = 0.0f;
  for (int s = 0; s < splits; ++s) v += partial[(static_cast<size_t>(s) * T + p) * N + o];
  const size_t dst = static_cast<size_t>(perm[p]) * N + o;
  if (y_bf16) static_cast<uint16_t*>(Y)[dst] = f32_to_bf16_bits(v);
  else static_cast<float*>(Y)[dst] = v;
}

}  // namespace

// ------------------------------------------------------------------ launchers
cudaError_t launch_route_stats(const void* X, bool x_bf16, const float* s_inv, const uint16_t* G, int T, int K,
                               int n_r, int qmax, int32_t* expert, float* sa, float* logits, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
#define QE_ROUTE(B, NR) k_route_stats<B, NR><<<T, 256, 0, st>>>(X, s_inv, G, T, K, n_r, qmax, expert, sa, logits)
  if (x_bf16) {
    if (n_r == 8) QE_ROUTE(true, 8);
    else if (n_r <= 4) QE_ROUTE(true, 4);
    else QE_ROUTE(true, 16);
  } else {
    if (n_r == 8) QE_ROUTE(false, 8);
    else if (n_r <= 4) QE_ROUTE(false, 4);
    else QE_ROUTE(false, 16);
  }
#undef QE_ROUTE
  return cudaGetLastError();
}

cudaError_t launch_bucket(const int32_t* expert, int T, int n_r, int32_t* perm, int32_t* pos, int32_t* offsets,
                          cudaStream_t st) {
  k_bucket<<<1, 1024, 0, st>>>(expert, T, n_r, perm, pos, offsets);
  return cudaGetLastError();
}

cudaError_t launch_act_quant(const void* X, bool x_bf16, const float* s_inv, int T, int K, int qmax,
                             const float* sa_tok, const int32_t* pos, int8_t* codes, float* sa_sorted,
                             uint16_t* act16, uint16_t* xb16, uint16_t* xlo16, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (x_bf16)
    k_act_quant<true><<<T, 256, 0, st>>>(X, s_inv, T, K, qmax, sa_tok, pos, codes, sa_sorted, act16, xb16, xlo16);
  else
    k_act_quant<false><<<T, 256, 0, st>>>(X, s_inv, T, K, qmax, sa_tok, pos, codes, sa_sorted, act16, xb16, xlo16);
  return cudaGetLastError();
}

cudaError_t launch_quantize_weights(const void* W, bool w_bf16, const float* s, int N, int K, int group,
                                    int w_bits, uint8_t* packed, void* w_scale, int s16, int* err,
                                    cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(ceil_div(N, kTileN)), static_cast<unsigned>(ceil_div(K, kTileK)));
  if (w_bits == 4) {
    if (w_bf16) k_quant_w<true, 4><<<grid, 128, 0, st>>>(W, s, N, K, group, packed, w_scale, s16, err);
    else k_quant_w<false, 4><<<grid, 128, 0, st>>>(W, s, N, K, group, packed, w_scale, s16, err);
  } else {
    if (w_bf16) k_quant_w<true, 3><<<grid, 128, 0, st>>>(W, s, N, K, group, packed, w_scale, s16, err);
    else k_quant_w<false, 3><<<grid, 128, 0, st>>>(W, s, N, K, group, packed, w_scale, s16, err);
  }
  return cudaGetLastError();
}

cudaError_t launch_colstats(const void* W, bool w_bf16, int N, int K, float* w_mean, float* w_colmax,
                            cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>(ceil_div(K, 64));
  if (w_bf16) k_colstats<true><<<grid, 64, 0, st>>>(W, N, K, w_mean, w_colmax);
  else k_colstats<false><<<grid, 64, 0, st>>>(W, N, K, w_mean, w_colmax);
  return cudaGetLastError();
}

cudaError_t launch_recip(const float* s, int K, float* s_inv, cudaStream_t st) {
  k_recip<<<static_cast<unsigned>(ceil_div(K, 256)), 256, 0, st>>>(s, K, s_inv);
  return cudaGetLastError();
}

cudaError_t launch_unpack_weights(const uint8_t* packed, int N, int K, int w_bits, int8_t* codes,
                                  cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(ceil_div(N, kTileN)), static_cast<unsigned>(ceil_div(K, kTileK)));
  if (w_bits == 4) k_unpack_w<4><<<grid, 128, 0, st>>>(packed, N, K, codes);
  else k_unpack_w<3><<<grid, 128, 0, st>>>(packed, N, K, codes);
  return cudaGetLastError();
}

cudaError_t launch_pack_adapters(const AdapterGeom& g, int K, int N, const uint16_t* A_s, const uint16_t* B_s,
                                 const uint16_t* A_r, const uint16_t* B_r, const uint16_t* G, const int32_t* channels,
                                 uint8_t* out, int* err, cudaStream_t st) {
  k_pack_adapters<<<592, 256, 0, st>>>(K, N, g.r_s, g.n_r, g.r_r > 0 ? g.r_r : 1, g.R_a, g.R_pad, g.R_tot, g.R_rt,
                                       g.kc, A_s, B_s, A_r, B_r, G, channels,
                                       reinterpret_cast<uint16_t*>(out + g.off_acat),
                                       reinterpret_cast<uint16_t*>(out + g.off_bcat),
                                       reinterpret_cast<int32_t*>(out + g.off_rch),
                                       reinterpret_cast<uint16_t*>(out + g.off_rar), err);
  return cudaGetLastError();
}

cudaError_t launch_split_f32(const float* X, const float* s_inv, int T, int K, uint16_t* xhi, uint16_t* xlo,
                             float* amax, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  k_split_f32<<<static_cast<unsigned>(ceil_div(T, 8)), 256, 0, st>>>(X, s_inv, T, K, xhi, xlo, amax);
  return cudaGetLastError();
}

constexpr int kRQMaxSmem = 220 * 1024;  // covers d_in <= 32768, R_pad <= 512, T <= 2^20

int route_quant_grid() {
  static int grid = 0;
  if (grid == 0) {
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return 0;
    if (cudaFuncSetAttribute(k_route_quant<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kRQMaxSmem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(k_route_quant<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kRQMaxSmem) !=
            cudaSuccess)
      return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_route_quant<true>, kRQThreads, kRQMaxSmem) !=
            cudaSuccess ||
        per_sm < 1)
      return 0;
    grid = std::min(sms, kRouteQuantMaxGrid);
  }
  return grid;
}

cudaError_t launch_route_quant(const RouteQuantParams& q, cudaStream_t st) {
  if (q.T == 0) return cudaSuccess;
  // one CTA per SM, or one per token when there are fewer tokens (decode)
  const int grid = std::min(route_quant_grid(), q.T);
  if (grid == 0) return cudaErrorInvalidConfiguration;
  RouteQuantArgs a{};
  a.partial = q.partial;
  a.nslots = q.nslots;
  a.R_tot = q.R_tot;
  a.R_pad = q.R_pad;
  a.R_rt = q.R_rt;
  a.kc = q.kc;
  a.rch = q.rch;
  a.rar = q.rar;
  a.n_r = q.n_r;
  a.r_s = q.r_s;
  a.r_r = q.r_r > 0 ? q.r_r : 1;
  a.R_a = q.R_a;
  a.X = q.X;
  a.s_inv = q.s_inv;
  a.amax = q.amax;
  a.T = q.T;
  a.K = q.K;
  a.qmax = q.qmax;
  a.chunk = static_cast<int>(ceil_div(q.T, grid));
  const size_t smem = route_quant_smem(q.K, a.chunk, q.R_pad);
  if (smem > static_cast<size_t>(kRQMaxSmem)) return cudaErrorInvalidValue;
  a.do_route = q.do_route;
  a.do_quant = q.do_quant;
  a.expert = q.expert;
  a.sa_tok = q.sa_tok;
  a.perm = q.perm;
  a.pos = q.pos;
  a.offsets = q.offsets;
  a.counts = q.counts;
  a.barrier = q.barrier;
  a.codes = q.codes;
  a.act16 = q.act16;
  a.sa_sorted = q.sa_sorted;
  a.ucat = q.ucat;
  a.su_sorted = q.su_sorted;
  a.zero_words = q.zero_words;
  a.n_zero_words = q.zero_words ? q.n_zero_words : 0;
  a.err = q.err;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kRQThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (q.x_bf16) return cudaLaunchKernelEx(&cfg, k_route_quant<true>, a);
  return cudaLaunchKernelEx(&cfg, k_route_quant<false>, a);
}

cudaError_t launch_splitk_reduce(const float* partial, int splits, const int32_t* perm, int T, int N, void* Y,
                                 int y_bf16, cudaStream_t st) {
  const size_t n = static_cast<size_t>(T) * N;
  if (n == 0) return cudaSuccess;
  k_splitk_reduce<<<static_cast<unsigned>(ceil_div(n, 256)), 256, 0, st>>>(partial, splits, perm, T, N, Y, y_bf16);
  return cudaGetLastError();
}

}  // namespace qe
