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

// marked_only: the CTAs stride over the tokens and take only those whose first index slot holds
// the mark -1 (left by k_topk_stream for rows it does not resolve).
template <bool BF16>
__global__ void __launch_bounds__(kTopkThreads) k_topk(const void* __restrict__ X, const float* __restrict__ w,
                                                       int T, int K, int k, int32_t* __restrict__ idx_out,
                                                       int32_t* __restrict__ hist, int marked_only) {
  extern __shared__ uint32_t keys[];  // [K]
  __shared__ int whist[kTopkWarps][256];
  __shared__ int digits[256];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_remaining;
  __shared__ int sgt[kTopkThreads], seq[kTopkThreads];
  __shared__ unsigned long long sel[128];
  __shared__ int mlist[kTopkThreads];
  __shared__ int s_nm;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int tb = blockIdx.x; tb < T; tb += gridDim.x * kTopkThreads) {
  int nm = 1;
  if (marked_only) {
    // this CTA's next kTopkThreads tokens, one per thread: list the marked ones
    __syncthreads();
    if (tid == 0) s_nm = 0;
    __syncthreads();
    const int tc = tb + tid * static_cast<int>(gridDim.x);
    if (tc < T && idx_out[static_cast<size_t>(tc) * k] < 0) mlist[atomicAdd(&s_nm, 1)] = tc;
    __syncthreads();
    nm = s_nm;
  }
  for (int q = 0; q < nm; ++q) {
  const int t = marked_only ? mlist[q] : tb;
  __syncthreads();  // shared memory of the previous token is free
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
  }
}

// ------------------------------------------------------------------ Top-k importance, streaming form
// bf16 rows with 7680 <= K <= 30720. Persistent CTAs (one per SM, 1024 threads) stride over the
// tokens, three row buffers in flight (untiled bulk copies). Warp roles, linked by mbarriers:
//  - scoring warps 0-29 hold the weight column means in registers (4 chunks of 8 channels per
//    thread). Per token: scores s = fl32(|x| * w); each thread keeps the maximum of each of its
//    chunks, and every warp publishes the j-th largest of its 32 lane maxima (j = ceil(k/30)),
//    a score that j distinct channels of the warp reach. After a barrier among the scoring
//    warps, each takes tau = the m-th largest of the 30 published values (m = ceil(k/j)): m
//    warps with j distinct channels each reach it, so at least k channels do, and every channel
//    of the Top-k set has s >= tau. The owners of the chunks whose maximum reaches tau list them
//    (channel base, 8 x values, 8 weights) in their warp's region of the token's list;
//  - selecting warps 30-31 take the tokens in turn: once a token's list is complete the warp
//    stages the token three steps ahead into the freed row buffer, scores the listed chunks again
//    and keeps the channels with s >= tau as 64-bit keys (score desc, channel asc). At most
//    kTSSel candidates are ranked among themselves by counting; more go through a bit-serial
//    threshold search (two bits per step, warp sums) on the score keys held in registers until
//    at most kTSSel remain. Ranks below k are the output slots.
// A row with more than kTSWarpCap listed chunks in one warp's region, more than kTSCap candidates
// or more than kTSSel at or above the final threshold (rows of mostly equal scores) is marked -1
// in its first slot and resolved by k_topk (marked_only).
constexpr int kTSThreads = 1024;
constexpr int kTSSelectors = 2;  // = list buffers
constexpr int kTSRowStages = 3;
constexpr int kTSScorerWarps = kTSThreads / 32 - kTSSelectors;
constexpr int kTSScorers = kTSScorerWarps * 32;
constexpr int kTSChunks = 4;  // channels (tid + 960 j) * 8 .. +7, j < 4
constexpr int kTSRegKeys = 12;  // score keys per lane held in registers by a selecting warp
constexpr int kTSCap = 32 * kTSRegKeys;
constexpr int kTSWarpCap = 12;  // listed chunks per scoring warp and token
constexpr int kTSListSlots = kTSScorerWarps * kTSWarpCap;
constexpr int kTSSel = 64;
constexpr int kTSMinK = kTSScorers * 8;
constexpr int kTSMaxK = kTSScorers * 8 * kTSChunks;

__device__ __forceinline__ unsigned long long topk_comp(float s, int c) {
  return (static_cast<unsigned long long>(order_key(s)) << 32) |
         static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(c));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// the 8 scores of one chunk (8 bf16 x values, 8 weights)
__device__ __forceinline__ void chunk_scores(const uint4 u, const float (&w8)[8], float (&sc)[8]) {
  const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    sc[2 * i] = __fmul_rn(fabsf(__uint_as_float(uu[i] << 16)), w8[2 * i]);
    sc[2 * i + 1] = __fmul_rn(fabsf(__uint_as_float(uu[i] & 0xFFFF0000u)), w8[2 * i + 1]);
  }
}

// Step 3 for one token, by one warp: candidates ck[0..nc) -> idx_out row t (+ hist).
__device__ __forceinline__ void topk_select(int t, const unsigned long long* ck, int nc, int k,
                                            int32_t* __restrict__ idx_out, int32_t* __restrict__ hist,
                                            unsigned long long* skey, int lane) {
  if (nc < k || nc > 32 * kTSRegKeys) {
    if (lane == 0) idx_out[static_cast<size_t>(t) * k] = -1;
    return;
  }
  if (nc <= kTSSel) {
    // few candidates: rank them all directly (ck is padded with zero keys to a multiple of 8)
    for (int q = lane; q < nc; q += 32) {
      const unsigned long long me = ck[q];
      int r = 0;
      for (int x = 0; x < nc; x += 8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) r += ck[x + u] > me ? 1 : 0;
      }
      if (r < k) {
        const int c = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(me & 0xFFFFFFFFull));
        idx_out[static_cast<size_t>(t) * k + r] = c;
        if (hist) atomicAdd(hist + c, 1);
      }
    }
    __syncwarp();
    return;
  }
  uint32_t key[kTSRegKeys];
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
  for (int r = 0; r < kTSRegKeys; ++r) {
    const int i = lane + 32 * r;
    key[r] = i < nc ? static_cast<uint32_t>(ck[i] >> 32) : 0u;  // 0 is below every score key
    if (i < nc) {
      kmin = min(kmin, key[r]);
      kmax = max(kmax, key[r]);
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  // Every key lies in [kmin, kmax], so the bits above the highest differing bit are kmax's.
  // Invariant: count(key >= v) >= k. Stop early once count <= kTSSel.
  uint32_t v = kmax;
  if (kmin != kmax) {
    int b = 31 - __clz(kmin ^ kmax);
    v = b == 31 ? 0u : (kmax & ~((2u << b) - 1u));
    int cv = nc;
    for (; b >= 1 && cv > kTSSel; b -= 2) {
      const uint32_t p1 = v | (1u << (b - 1)), p2 = v | (2u << (b - 1)), p3 = v | (3u << (b - 1));
      int c1 = 0, c2 = 0, c3 = 0;
#pragma unroll
      for (int r = 0; r < kTSRegKeys; ++r) {
        c1 += key[r] >= p1 ? 1 : 0;
        c2 += key[r] >= p2 ? 1 : 0;
        c3 += key[r] >= p3 ? 1 : 0;
      }
      c1 = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c1)));
      c2 = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c2)));
      c3 = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c3)));
      if (c3 >= k) {
        v = p3;
        cv = c3;
      } else if (c2 >= k) {
        v = p2;
        cv = c2;
      } else if (c1 >= k) {
        v = p1;
        cv = c1;
      }
    }
    if (b == 0 && cv > kTSSel) {
      int c1 = 0;
#pragma unroll
      for (int r = 0; r < kTSRegKeys; ++r) c1 += key[r] >= (v | 1u) ? 1 : 0;
      if (static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c1))) >= k) v |= 1u;
    }
  }
  // the set S = {score key >= v} (k of them at least): compact, rank by counting within S
  int ns = 0;
#pragma unroll
  for (int r = 0; r < kTSRegKeys; ++r) {
    const int i = lane + 32 * r;
    const bool in = i < nc && key[r] >= v;
    const uint32_t bal = __ballot_sync(0xffffffffu, in);
    const int at = ns + __popc(bal & ((1u << lane) - 1u));
    if (in && at < kTSSel) skey[at] = ck[i];
    ns += __popc(bal);
  }
  if (ns > kTSSel) {
    if (lane == 0) idx_out[static_cast<size_t>(t) * k] = -1;
    return;
  }
  for (int x = ns + lane; x < ((ns + 7) & ~7); x += 32) skey[x] = 0ull;  // pad to a multiple of 8
  __syncwarp();
  for (int q = lane; q < ns; q += 32) {
    const unsigned long long me = skey[q];
    int r = 0;
    for (int x = 0; x < ns; x += 8) {
#pragma unroll
      for (int u = 0; u < 8; ++u) r += skey[x + u] > me ? 1 : 0;
    }
    if (r < k) {
      const int c = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(me & 0xFFFFFFFFull));
      idx_out[static_cast<size_t>(t) * k + r] = c;
      if (hist) atomicAdd(hist + c, 1);
    }
  }
  __syncwarp();
}

// A bounded wait that also gives up once another thread of the CTA has given up.
__device__ __forceinline__ bool ts_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (!mbar_try_wait(bar, parity)) {
    // back off: a waiting warp leaves its issue slots to the warps it waits for
    __nanosleep(spins < 4 ? 32 : 128);
    if ((++spins & 15u) == 0u) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        record_error(err, DEVERR_WAIT_PRODUCER);
        *abort_flag = 1;
        return false;
      }
    }
  }
  return true;
}

// Barrier 1 over the scoring warps; returns whether any of them passed pred = true.
__device__ __forceinline__ bool scorers_sync_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "n"(kTSScorers)
      : "memory");
  return r != 0;
}

struct TSList {
  uint4 x[kTSListSlots];      // the chunk's 8 bf16 x values
  float4 w[kTSListSlots][2];  // its 8 weights
  int16_t ci[kTSListSlots];   // chunk index (channel base / 8)
  int count[32];              // listed chunks per scoring warp (kTSWarpCap + 1: overflow)
};

__global__ void __launch_bounds__(kTSThreads, 1) k_topk_stream(const uint16_t* __restrict__ X,
                                                               const float* __restrict__ w, int T, int K, int k,
                                                               int32_t* __restrict__ idx_out,
                                                               int32_t* __restrict__ hist, int* err) {
  extern __shared__ __align__(128) uint8_t tsm[];
  uint16_t* rows = reinterpret_cast<uint16_t*>(tsm);  // [3][K]
  TSList* lists = reinterpret_cast<TSList*>(tsm + kTSRowStages * K * 2);  // [2]
  __shared__ unsigned long long ckey[kTSSelectors][kTSCap + 8];
  __shared__ unsigned long long skey[kTSSelectors][kTSSel + 8];
  __shared__ int16_t sq[kTSSelectors][kTSListSlots];
  __shared__ float wthr[kTSSelectors][32];
  __shared__ __align__(8) uint64_t row_full[kTSRowStages], list_full[kTSSelectors], list_empty[kTSSelectors];
  __shared__ int issued[kTSRowStages], consumed[kTSRowStages];
  __shared__ int s_abort;
  volatile int* abort_flag = &s_abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t row_bytes = static_cast<uint32_t>(K) * 2u;
  const int G = static_cast<int>(gridDim.x);
  const int KC = K / 8;
  const int jj = (k + kTSScorerWarps - 1) / kTSScorerWarps;  // order statistic per warp
  const int mm = (k + jj - 1) / jj;                           // warps combined, <= 30
  if (tid == 0) {
    for (int r = 0; r < kTSRowStages; ++r) {
      mbar_init(&row_full[r], 1);
      issued[r] = 0;
      consumed[r] = 0;
    }
    for (int l = 0; l < kTSSelectors; ++l) {
      mbar_init(&list_full[l], kTSScorerWarps);
      mbar_init(&list_empty[l], 1);
    }
    s_abort = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (tid == 0) {
    for (int r = 0; r < kTSRowStages; ++r) {
      const int t = blockIdx.x + r * G;
      if (t < T) {
        issued[r] = 1;
        mbar_arrive_expect_tx(&row_full[r], row_bytes);
        bulk_load(rows + r * K, X + static_cast<size_t>(t) * K, row_bytes, &row_full[r]);
      }
    }
  }
  if (warp < kTSScorerWarps) {
    // ---------------- scoring warps
    float wr[kTSChunks][8];
#pragma unroll
    for (int j = 0; j < kTSChunks; ++j) {
      const int c0 = (tid + kTSScorers * j) * 8;
      if (c0 < K) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(w + c0));
        const float4 b = __ldg(reinterpret_cast<const float4*>(w + c0) + 1);
        wr[j][0] = a.x; wr[j][1] = a.y; wr[j][2] = a.z; wr[j][3] = a.w;
        wr[j][4] = b.x; wr[j][5] = b.y; wr[j][6] = b.z; wr[j][7] = b.w;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) wr[j][i] = 0.0f;
      }
    }
    int it = 0;
    for (int t = blockIdx.x; t < T; t += G, ++it) {
      const int r = it % kTSRowStages, l = it & 1;
      bool ok = ts_wait(&row_full[r], static_cast<uint32_t>((it / kTSRowStages) & 1), abort_flag, err);
      if (ok && tid == 0) consumed[r] += 1;
      if (ok && it >= kTSSelectors) ok = ts_wait(&list_empty[l], static_cast<uint32_t>(((it >> 1) - 1) & 1), abort_flag, err);
      const uint16_t* row = rows + r * K;
      float cmax[kTSChunks];
      float m = -INFINITY;
#pragma unroll
      for (int j = 0; j < kTSChunks; ++j) {
        const int ci = tid + kTSScorers * j;
        cmax[j] = -INFINITY;
        if (ci < KC) {
          float sc[8];
          chunk_scores(*reinterpret_cast<const uint4*>(row + ci * 8), wr[j], sc);
          cmax[j] = fmaxf(fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3])),
                          fmaxf(fmaxf(sc[4], sc[5]), fmaxf(sc[6], sc[7])));
          m = fmaxf(m, cmax[j]);
        }
      }
      float tw = warp_max(m);
      for (int q = 1; q < jj; ++q) {
        // drop one lane holding the current maximum, take the maximum of the rest
        const uint32_t holder = __ballot_sync(0xffffffffu, m == tw);
        if (lane == __ffs(holder) - 1) m = -INFINITY;
        tw = warp_max(m);
      }
      if (lane == 0) wthr[l][warp] = tw;
      if (scorers_sync_or(!ok)) break;  // every warp's value is published (or a wait gave up)
      // tau = the mm-th largest of the 30 published values (a sort across the lanes)
      float v = lane < kTSScorerWarps ? wthr[l][lane] : -INFINITY;
#pragma unroll
      for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          const float o = __shfl_xor_sync(0xffffffffu, v, stride);
          const bool desc = (lane & size) == 0 || size == 32;
          v = (((lane & stride) == 0) == desc) ? fmaxf(v, o) : fminf(v, o);
        }
      }
      const float tau = __shfl_sync(0xffffffffu, v, mm - 1);
      // list the chunks that reach tau in this warp's region
      TSList& L = lists[l];
      int wc = 0;
#pragma unroll
      for (int j = 0; j < kTSChunks; ++j) {
        const bool cand = cmax[j] >= tau;
        const uint32_t bal = __ballot_sync(0xffffffffu, cand);
        if (cand) {
          const int at = wc + __popc(bal & ((1u << lane) - 1u));
          if (at < kTSWarpCap) {
            const int slot = warp * kTSWarpCap + at;
            const int ci = tid + kTSScorers * j;
            L.ci[slot] = static_cast<int16_t>(ci);
            L.x[slot] = *reinterpret_cast<const uint4*>(row + ci * 8);
            L.w[slot][0] = make_float4(wr[j][0], wr[j][1], wr[j][2], wr[j][3]);
            L.w[slot][1] = make_float4(wr[j][4], wr[j][5], wr[j][6], wr[j][7]);
          }
        }
        wc += __popc(bal);
      }
      if (lane == 0) L.count[warp] = wc > kTSWarpCap ? kTSWarpCap + 1 : wc;
      __syncwarp();
      if (lane == 0) mbar_arrive(&list_full[l]);
    }
  } else {
    // ---------------- selecting warps: warp 30 + l takes the tokens with it % 2 == l
    const int l = warp - kTSScorerWarps;
    for (int it = l, t = blockIdx.x + l * G; t < T; it += kTSSelectors, t += kTSSelectors * G) {
      if (!ts_wait(&list_full[l], static_cast<uint32_t>((it >> 1) & 1), abort_flag, err)) break;
      if (lane == 0) {
        // every scoring warp is done with this row: stage the token three steps ahead into it
        const int r = it % kTSRowStages;
        const int t3 = t + kTSRowStages * G;
        if (t3 < T) {
          atomicAdd(&issued[r], 1);  // both selecting warps fill this buffer over time
          mbar_arrive_expect_tx(&row_full[r], row_bytes);
          bulk_load(rows + r * K, X + static_cast<size_t>(t3) * K, row_bytes, &row_full[r]);
        }
      }
      const TSList& L = lists[l];
      // the same tau as the scoring warps
      float v = lane < kTSScorerWarps ? wthr[l][lane] : -INFINITY;
#pragma unroll
      for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          const float o = __shfl_xor_sync(0xffffffffu, v, stride);
          const bool desc = (lane & size) == 0 || size == 32;
          v = (((lane & stride) == 0) == desc) ? fmaxf(v, o) : fminf(v, o);
        }
      }
      const float tau = __shfl_sync(0xffffffffu, v, mm - 1);
      // gather the listed chunks: warp region counts -> one index list
      const int cnt = lane < kTSScorerWarps ? L.count[lane] : 0;
      const bool overflow = __any_sync(0xffffffffu, cnt > kTSWarpCap);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int nch = overflow ? 0 : __shfl_sync(0xffffffffu, incl, 31);
      if (!overflow)
        for (int e = 0; e < cnt; ++e) sq[l][incl - cnt + e] = static_cast<int16_t>(lane * kTSWarpCap + e);
      __syncwarp();
      int nc = overflow ? kTSCap + 1 : 0;
      for (int q0 = 0; q0 < nch; q0 += 32) {
        const int qq = q0 + lane;
        uint32_t m8 = 0u;
        float sc[8];
        int c0 = 0;
        if (qq < nch) {
          const int q = sq[l][qq];
          c0 = static_cast<int>(L.ci[q]) * 8;
          const float4 wa = L.w[q][0], wb = L.w[q][1];
          const float w8[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
          chunk_scores(L.x[q], w8, sc);
#pragma unroll
          for (int i = 0; i < 8; ++i) m8 |= (sc[i] >= tau ? 1u : 0u) << i;
        }
        const int c = __popc(m8);
        int ic = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, ic, o);
          if (lane >= o) ic += y;
        }
        int p = nc + ic - c;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if ((m8 >> i) & 1u) {
            if (p < kTSCap) ckey[l][p] = topk_comp(sc[i], c0 + i);
            ++p;
          }
        }
        nc += __shfl_sync(0xffffffffu, ic, 31);
      }
      // zero keys up to a multiple of 8 for the unrolled ranking
      if (nc <= kTSCap && lane < ((nc + 7) & ~7) - nc) ckey[l][nc + lane] = 0ull;
      __syncwarp();
      if (lane == 0) mbar_arrive(&list_empty[l]);  // the list buffer is free for token it + 2
      topk_select(t, ckey[l], nc, k, idx_out, hist, skey[l], lane);
    }
  }
  __syncthreads();
  if (tid == 0 && s_abort) {
    // a wait gave up: let every copy still in flight land before the CTA exits
    for (int r = 0; r < kTSRowStages; ++r)
      if (issued[r] > consumed[r])
        mbar_wait_for(&row_full[r], static_cast<uint32_t>(consumed[r] & 1), nullptr, 0, kDrainLimitNs);
  }
}

// ------------------------------------------------------------------ channel split by frequency
// Ranks channels by calibration count (higher first, equal counts by lower index). Rank r in
// [k, k + C) gets position r - k; every other channel gets -1. One CTA, the counts staged in
// shared memory as order-preserving keys when they fit: a radix select (4 passes
// of 8 bits over order-preserving keys) finds the count v* of the n-th ranked channel,
// n = min(k + C, d); one pass in index order then compacts the channels above v* and numbers
// the ties at v* by block scans; the channels above v* (fewer than n) are ranked among
// themselves by counting.
constexpr int kSplitThreads = 1024;
constexpr int kSplitMaxSel = 4096 + 128;
constexpr int kSplitStageMax = 36864;  // counts staged in shared memory up to this many channels (144 KB)

__device__ __forceinline__ uint32_t split_key(int32_t v) { return static_cast<uint32_t>(v) ^ 0x80000000u; }

// exclusive scan of v over the block (kSplitThreads threads); *total gets the block sum
__device__ __forceinline__ int split_block_scan(int v, int* wt, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wt[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int t = wt[lane];
    int sc = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, sc, o);
      if (lane >= o) sc += y;
    }
    wt[lane] = sc - t;
    if (lane == 31) wt[32] = sc;
  }
  __syncthreads();
  const int ex = wt[warp] + x - v;
  *total = wt[32];
  __syncthreads();
  return ex;
}

// keys of the counts: staged in shared memory when they fit (staged != 0), else read from hist
__device__ __forceinline__ uint32_t split_key_at(const int32_t* __restrict__ hist, const uint32_t* sk, bool staged,
                                                 int c) {
  return staged ? sk[c] : split_key(hist[c]);
}

__global__ void __launch_bounds__(kSplitThreads) k_split_channels(const int32_t* __restrict__ hist, int d, int k,
                                                                   int C, int32_t* __restrict__ pos, int staged) {
  extern __shared__ uint32_t split_dyn[];  // per-warp digit counts [32][256], then the keys [d] when staged
  int (*wbins)[256] = reinterpret_cast<int (*)[256]>(split_dyn);
  uint32_t* sk = split_dyn + (kSplitThreads / 32) * 256;
  __shared__ int bins[256];
  __shared__ int wt[33];
  __shared__ uint32_t s_prefix, s_kmin, s_kmax;
  __shared__ int s_rem;
  __shared__ int a_idx[kSplitMaxSel];
  __shared__ uint32_t a_key[kSplitMaxSel];
  int* a_rank = &wbins[0][0];  // reused once the radix passes are done (8192 >= kSplitMaxSel)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = min(k + C, d);
  if (tid == 0) {
    s_kmin = 0xFFFFFFFFu;
    s_kmax = 0u;
  }
  __syncthreads();
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll 8
  for (int c = tid; c < d; c += kSplitThreads) {
    const uint32_t u = split_key(__ldg(hist + c));
    if (staged) sk[c] = u;
    lo = min(lo, u);
    hi = max(hi, u);
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  if (lane == 0) {
    atomicMin(&s_kmin, lo);
    atomicMax(&s_kmax, hi);
  }
  __syncthreads();
  // radix select of the n-th largest key, from the highest byte in which the keys differ
  const uint32_t kdiff = s_kmin ^ s_kmax;
  int shift = kdiff == 0u ? 0 : ((31 - __clz(kdiff)) / 8) * 8;
  uint32_t mask = shift == 24 ? 0u : ~((1u << (shift + 8)) - 1u);
  uint32_t prefix = s_kmax & mask;
  int rem = n;
  for (; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSplitThreads) bins[i] = 0;
    for (int i = lane; i < 256; i += 32) wbins[warp][i] = 0;
    __syncthreads();
    for (int base = 0; base < d; base += kSplitThreads) {
      const int c = base + tid;
      const uint32_t u = c < d ? split_key_at(hist, sk, staged, c) : 0u;
      const bool match = c < d && (u & mask) == prefix;
      const uint32_t active = __ballot_sync(0xffffffffu, match);
      if (match) {
        const int dg = static_cast<int>((u >> shift) & 255u);
        const int lead = __ffs(active) - 1;
        const int d0 = __shfl_sync(active, dg, lead);
        // counts mostly share their high bits: one add when the whole warp has one digit
        if (__all_sync(active, dg == d0)) {
          if (lane == lead) atomicAdd(&bins[dg], __popc(active));
        } else {
          atomicAdd(&wbins[warp][dg], 1);
        }
      }
    }
    __syncthreads();
    if (tid < 256) {
      int sum = bins[tid];
#pragma unroll 8
      for (int w2 = 0; w2 < kSplitThreads / 32; ++w2) sum += wbins[w2][tid];
      bins[tid] = sum;
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits 255-8l .. 248-8l (descending); find where the count from the top
      // reaches rem
      int cnt[8];
      int lsum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[j] = bins[255 - 8 * lane - j];
        lsum += cnt[j];
      }
      int incl = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int excl = incl - lsum;
      const uint32_t hm = __ballot_sync(0xffffffffu, excl < rem && incl >= rem);
      if (lane == __ffs(hm) - 1) {
        int run = excl, dg = 255 - 8 * lane - 7;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (run + cnt[j] >= rem) {
            dg = 255 - 8 * lane - j;
            break;
          }
          run += cnt[j];
        }
        s_prefix = prefix | (static_cast<uint32_t>(dg) << shift);
        s_rem = rem - run;
      }
    }
    __syncthreads();
    prefix = s_prefix;
    rem = s_rem;
    mask |= 255u << shift;
    __syncthreads();
  }
  // prefix = key of v*; n - rem channels lie above it, the first rem ties (by index) are taken.
  // Each thread takes a contiguous range of channels, so one block scan orders them by index.
  const int nA = n - rem;
  const int per = (d + kSplitThreads - 1) / kSplitThreads;
  const int c_lo = min(d, tid * per), c_hi = min(d, c_lo + per);
  int na = 0, nb = 0;
  for (int c = c_lo; c < c_hi; ++c) {
    const uint32_t u = split_key_at(hist, sk, staged, c);
    na += u > prefix ? 1 : 0;
    nb += u == prefix ? 1 : 0;
  }
  int tot;
  int ia = split_block_scan(na, wt, &tot);
  int ib = split_block_scan(nb, wt, &tot);
  for (int c = c_lo; c < c_hi; ++c) {
    const uint32_t u = split_key_at(hist, sk, staged, c);
    int p = -1;
    if (u > prefix) {
      a_idx[ia] = c;
      a_key[ia] = u;
      ++ia;
      continue;
    }
    if (u == prefix) {
      if (ib < rem && nA + ib >= k) p = nA + ib - k;
      ++ib;
    }
    pos[c] = p;
  }
  // ranks of the channels above v* by counting: candidate i = tid % nap against slice tid / nap
  // of the list (partial counts added in shared memory)
  for (int i = tid; i < nA; i += kSplitThreads) a_rank[i] = 0;
  __syncthreads();
  const int nap = (nA + 31) & ~31;
  if (nap > 0) {
    const int P = nap <= kSplitThreads ? kSplitThreads / nap : 1;
    for (int i0 = 0; i0 < nA; i0 += kSplitThreads) {
      const int i = i0 + (P > 1 ? tid % nap : tid), part = P > 1 ? tid / nap : 0;
      if (i < nA && part < P) {
        const uint32_t u = a_key[i];
        const int c = a_idx[i];
        const int j0 = part * nA / P, j1 = (part + 1) * nA / P;
        int r = 0;
#pragma unroll 4
        for (int j = j0; j < j1; ++j) {
          const uint32_t uj = a_key[j];
          r += (uj > u || (uj == u && a_idx[j] < c)) ? 1 : 0;
        }
        atomicAdd(&a_rank[i], r);
      }
      if (P > 1) break;
    }
  }
  __syncthreads();
  for (int i = tid; i < nA; i += kSplitThreads) {
    const int r = a_rank[i];
    pos[a_idx[i]] = r >= k ? r - k : -1;
  }
}

// ------------------------------------------------------------------ co-occurrence and NPMI
// O[i][j] = number of tokens whose Top-k set holds both token-dependent channels i and j.
// CTA (row block of RB rows, token chunk): the block's RB x C counters live in shared memory.
// The chunk's index rows are staged in batches, mapped through channel_pos to positions (int16,
// -1 for other channels) by all threads at once. A warp then takes a token with its positions in
// lane registers; for every position inside the row block (a ballot) it adds 1 to that counter
// row at each of the token's positions (shared-memory atomics). The block finally adds its counts
// to O with integer atomics, so the result does not depend on the schedule.
constexpr int kCoocThreads = 512;
constexpr int kCoocWarps = kCoocThreads / 32;
constexpr int kCoocCounters = 16384;  // 64 KB of counters per CTA
constexpr int kCoocStage = 16384;     // staged positions per batch (32 KB)

__global__ void __launch_bounds__(kCoocThreads) k_cooc(const int32_t* __restrict__ idx, int T, int k,
                                                        const int32_t* __restrict__ pos, int d_in, int C, int RB,
                                                        int tokens_per_cta, int32_t* __restrict__ O) {
  extern __shared__ __align__(16) int cnt[];  // [RB][C], then int16 positions [batch][k]
  int16_t* qs = reinterpret_cast<int16_t*>(cnt + RB * C);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = blockIdx.x * RB;
  const int rows = min(RB, C - r0);
  const int t0 = blockIdx.y * tokens_per_cta, t1 = min(T, t0 + tokens_per_cta);
  const int batch = kCoocStage / k;
  for (int i = threadIdx.x; i < RB * C; i += kCoocThreads) cnt[i] = 0;
  for (int tb = t0; tb < t1; tb += batch) {
    const int nb = min(batch, t1 - tb);
    __syncthreads();  // counters zeroed / previous batch consumed
    const int32_t* src = idx + static_cast<size_t>(tb) * k;
    for (int e = threadIdx.x; e < nb * k; e += kCoocThreads) {
      const int c = src[e];
      int m = -1;
      if (c >= 0 && c < d_in) m = pos[c];
      qs[e] = static_cast<int16_t>((m >= 0 && m < C) ? m : -1);
    }
    __syncthreads();
    for (int tt = warp; tt < nb; tt += kCoocWarps) {
      const int16_t* q = qs + tt * k;
      int v[4];
#pragma unroll
      for (int s4 = 0; s4 < 4; ++s4) v[s4] = (lane + 32 * s4 < k) ? q[lane + 32 * s4] : -1;
#pragma unroll
      for (int s4 = 0; s4 < 4; ++s4) {
        if (32 * s4 >= k) break;
        uint32_t hb = __ballot_sync(0xffffffffu, v[s4] >= r0 && v[s4] < r0 + rows);
        while (hb) {
          const int la = __ffs(hb) - 1;
          hb &= hb - 1;
          int* crow = cnt + (__shfl_sync(0xffffffffu, v[s4], la) - r0) * C;
#pragma unroll
          for (int s2 = 0; s2 < 4; ++s2)
            if (v[s2] >= 0) atomicAdd(crow + v[s2], 1);
        }
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < rows * C; i += kCoocThreads)
    if (cnt[i]) atomicAdd(&O[static_cast<size_t>(r0) * C + i], cnt[i]);
}

// S[i][j] = NPMI of channels i and j, in fp64 before the final rounding: p(i) = O[i][i] / T,
// p(i,j) = O[i][j] / T, S = ln(p(i,j) / (p(i) p(j))) / (-ln p(i,j)); -1 where the pair never
// co-occurs, 1 where it is in every token; entries below threshold -> 0 when threshold > -1.
__global__ void k_npmi(const int32_t* __restrict__ O, int C, int T, float threshold, float* __restrict__ S) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= C * C) return;
  const int i = e / C, j = e % C;
  const double inv_t = 1.0 / static_cast<double>(T);
  const double pij = O[e] * inv_t;
  double v;
  if (pij <= 0.0) {
    v = -1.0;
  } else if (pij >= 1.0) {
    v = 1.0;
  } else {
    const double pi = O[static_cast<size_t>(i) * C + i] * inv_t, pj = O[static_cast<size_t>(j) * C + j] * inv_t;
    v = log(pij / (pi * pj)) / (-log(pij));
  }
  if (threshold > -1.0f && v < static_cast<double>(threshold)) v = 0.0;
  S[e] = static_cast<float>(v);
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
                        int32_t* hist, int* err, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const size_t smem = static_cast<size_t>(K) * 4;
  cudaError_t e;
  if (x_bf16 && K >= kTSMinK && K <= kTSMaxK) {
    static int n_sm = 0;
    if (n_sm == 0) {
      int dev = 0;
      if (cudaGetDevice(&dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        n_sm = 148;
    }
    const int grid = std::min(T, n_sm);
    const size_t smem_s = static_cast<size_t>(K) * 2 * kTSRowStages + sizeof(TSList) * kTSSelectors;
    e = cudaFuncSetAttribute(k_topk_stream, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_s));
    if (e != cudaSuccess) return e;
    k_topk_stream<<<grid, kTSThreads, smem_s, st>>>(static_cast<const uint16_t*>(X), w_mean, T, K, k, idx, hist,
                                                    err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // rows the streaming pass left unresolved (marked -1)
    e = cudaFuncSetAttribute(k_topk<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k_topk<true><<<grid, kTopkThreads, smem, st>>>(X, w_mean, T, K, k, idx, hist, 1);
  } else if (x_bf16) {
    e = cudaFuncSetAttribute(k_topk<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k_topk<true><<<T, kTopkThreads, smem, st>>>(X, w_mean, T, K, k, idx, hist, 0);
  } else {
    e = cudaFuncSetAttribute(k_topk<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k_topk<false><<<T, kTopkThreads, smem, st>>>(X, w_mean, T, K, k, idx, hist, 0);
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

namespace qe {
cudaError_t launch_split_channels(const int32_t* hist, int d, int k, int C, int32_t* pos, cudaStream_t st) {
  const int staged = d <= kSplitStageMax ? 1 : 0;
  const size_t smem = static_cast<size_t>(kSplitThreads / 32) * 256 * 4 + (staged ? static_cast<size_t>(d) * 4 : 0);
  const cudaError_t e0 =
      cudaFuncSetAttribute(k_split_channels, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e0 != cudaSuccess) return e0;
  k_split_channels<<<1, kSplitThreads, smem, st>>>(hist, d, k, C, pos, staged);
  return cudaGetLastError();
}

cudaError_t launch_cooc_npmi(const int32_t* idx, int T, int k, const int32_t* pos, int d_in, int C, int32_t* O,
                             float* S, float threshold, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(O, 0, static_cast<size_t>(C) * C * sizeof(int32_t), st);
  if (e != cudaSuccess) return e;
  if (T > 0) {
    // about 16 row blocks: each CTA re-reads its chunk's index rows (cheap), and every token chunk
    // costs one global add per counter, so about one CTA per SM with long chunks
    const int RB = std::max(1, std::min(static_cast<int>(ceil_div(C, 16)), kCoocCounters / C));
    const int nrb = static_cast<int>(ceil_div(C, RB));
    int chunks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(ceil_div(148, nrb), ceil_div(T, 64))));
    const int tpc = static_cast<int>(ceil_div(T, chunks));
    chunks = static_cast<int>(ceil_div(T, tpc));
    const size_t smem = static_cast<size_t>(RB) * C * sizeof(int) + kCoocStage * sizeof(int16_t);
    e = cudaFuncSetAttribute(k_cooc, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k_cooc<<<dim3(static_cast<unsigned>(nrb), static_cast<unsigned>(chunks)), kCoocThreads, smem, st>>>(
        idx, T, k, pos, d_in, C, RB, tpc, O);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (S && T > 0) {
    const int n = C * C;
    k_npmi<<<static_cast<unsigned>(ceil_div(n, 256)), 256, 0, st>>>(O, C, T, threshold, S);
    e = cudaGetLastError();
  }
  return e;
}
}  // namespace qe
