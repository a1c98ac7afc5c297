// Tensor-core kernels (tcgen05 + TMEM + TMA) of the QE linear layer.
//
// k_qgemm: the main W4 x A8/A6 product with the QE epilogue. The tile is
//   M = 128 output channels (weights are the A operand, so each TMEM lane is
//   one output row) by N = BN token positions in bucket order (the B
//   operand). Each pipeline stage covers 128 input channels:
//     warp 0      TMA producer: activation codes (tensor map, 128B swizzle),
//                 plus one bulk copy of the 8 KB packed-int4 weight block
//     warps 2-3   unpack the int4 block into int8 in the 128B-swizzled A layout
//     warp 1      one elected thread issues tcgen05.mma kind::i8, one TMEM
//                 accumulator buffer per quantization group (double-buffered)
//     warps 4-11  epilogue: the per-group promotion acc += sw[o,j] * float(int32)
//                 in registers, then * sa[t], + adapter MMA result, and a
//                 scatter of the row to token order
//   Integer -> float without a convert instruction: every TMEM accumulator
//   starts at the bit pattern of 1.5*2^23. The int32 MMA adds the exact group
//   sum (|sum| < 2^22) onto it, so the value reads as the float
//   1.5*2^23 + sum, and one fp32 subtraction recovers the sum exactly.
//   After the last group, the stage ring carries the adapter operands:
//   B_catT (shared ++ routed up-projections, fp16) as A, and U_cat (the
//   bucket-ordered, expert-masked down-projections, fp16 with a per-token
//   power-of-two scale su) as B. An fp16 MMA puts them into a TMEM buffer,
//   and the epilogue adds it times su.
//
// k_ugemm: the adapter down-projection U = X . [A_s | A_r[0..N_r)] as a split-K
//   bf16 tcgen05 GEMM (M = 128 tokens, N = adapter columns) with fp32 partials.
#include <cuda_bf16.h>

#include <algorithm>

#include "qe_internal.h"
#include "qe_ptx.cuh"

namespace qe {
namespace {

constexpr uint32_t kMagicBits = 0x4B400000u;  // fp32 bit pattern of 1.5 * 2^23
constexpr float kMagic = 12582912.0f;

__device__ __forceinline__ uint32_t sext_nibbles(uint32_t x) {
  // x holds 4 nibbles in the low 4 bits of each byte; sign-extend each to a byte.
  return x | ((x & 0x08080808u) * 0x1Eu);
}

__device__ __forceinline__ uint16_t f2bf(float v) {
  __nv_bfloat16 h = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t*>(&h);
}

template <int BN>
struct QCfg {
  static constexpr int kA = 16384;                 // 128 rows x 128 B (int8 K=128 or bf16 K=64)
  static constexpr int kB = BN * 128;
  static constexpr int kWP = kW4BlockBytes;         // packed int4 block
  static constexpr int kStage = kA + kB + kWP;
  static constexpr int kStages = (BN >= 256) ? 3 : (BN >= 128 ? 4 : (BN >= 64 ? 5 : 6));
  static constexpr int kTmemCols = (2 * BN <= 32) ? 32 : 2 * BN;  // power of two for BN in {16..256}
  static constexpr int kCPT = BN / 2;              // columns per epilogue thread
  static constexpr int kChunk = (kCPT >= 32) ? 32 : kCPT;
  static constexpr size_t kSmem = 1024 /*align slack*/ + size_t(kStages) * kStage + 1024 /*barriers etc*/ +
                                  size_t(BN) * 12 /*sa + su + perm*/;
};

template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&v)[N]) {
  if constexpr (N == 32) tmem_ld32(taddr, v);
  else if constexpr (N == 16) tmem_ld16(taddr, v);
  else tmem_ld8(taddr, v);
}
template <int N>
__device__ __forceinline__ void tmem_fill(uint32_t taddr, uint32_t x) {
  if constexpr (N == 32) tmem_fill32(taddr, x);
  else if constexpr (N == 16) tmem_fill16(taddr, x);
  else tmem_fill8(taddr, x);
}

template <int BN, bool DBG>
__global__ void __launch_bounds__(384, 1)
    k_qgemm(const __grid_constant__ CUtensorMap tm_xq, const __grid_constant__ CUtensorMap tm_bcat,
            const __grid_constant__ CUtensorMap tm_ucat, const QgemmArgs a) {
  using C = QCfg<BN>;
  constexpr int NS = C::kStages;
  int* const a_err = a.err;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NS * C::kStage);
  uint64_t* full = bars;            // [NS] TMA bytes landed
  uint64_t* afull = bars + NS;      // [NS] unpack done (2 warp arrivals)
  uint64_t* empty = bars + 2 * NS;  // [NS] MMAs done reading the stage
  uint64_t* accf = bars + 3 * NS;   // [2] accumulator buffer ready for the epilogue
  uint64_t* acce = accf + 2;        // [2] accumulator buffer drained (8 warp arrivals)
  uint64_t* done = acce + 2;        // [1] teardown
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  float* sa_s = reinterpret_cast<float*>(smem + NS * C::kStage + 512);
  float* su_s = sa_s + BN;
  int32_t* perm_s = reinterpret_cast<int32_t*>(su_s + BN);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = blockIdx.x, o0 = nt * kTileN, p0 = blockIdx.y * BN, split = blockIdx.z;
  const int kb_begin = split * a.kb_per_split;
  const int kb_end = min(a.KB, kb_begin + a.kb_per_split);
  const int nkb = max(0, kb_end - kb_begin);
  const int n_ad = (split == 0) ? a.adapter_atoms : 0;
  const int n_iters = nkb + n_ad;
  const int gpb = kTileK / a.group;  // groups per 128-channel block
  const int G_total = a.K / a.group;
  // groups handled by this split
  const int g_begin = kb_begin * gpb;
  const int g_end = min(G_total, kb_end * gpb);
  const int n_groups = max(0, g_end - g_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&afull[s], 2);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 8);
    }
    mbar_init(done, 1);
    mbar_fence_init();
    prefetch_tmap(&tm_xq);
    if (n_ad) {
      prefetch_tmap(&tm_bcat);
      prefetch_tmap(&tm_ucat);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 4) {
    // epilogue threads: stage sa/perm of the tile, put the magic bias in both buffers
    const int et = threadIdx.x - 128;
    for (int c = et; c < BN; c += 256) {
      const int p = p0 + c;
      sa_s[c] = (p < a.T) ? a.sa_sorted[p] : 0.0f;
      su_s[c] = (p < a.T && a.su_sorted) ? a.su_sorted[p] : 0.0f;
      perm_s[c] = (p < a.T) ? a.perm[p] : -1;
    }
    const int q = warp & 3, h = (warp - 4) >> 2;
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int c = 0; c < C::kCPT; c += C::kChunk)
        tmem_fill<C::kChunk>(tmem + (static_cast<uint32_t>(32 * q) << 16) + b * BN + h * C::kCPT + c, kMagicBits);
    tmem_wait_st();
    tc_fence_before();
  }
  __syncthreads();
  // Register split (launch: 384 x 168 = 64512): the producer/MMA/unpack
  // warpgroup gives back to 56, and the two epilogue warpgroups take 224 each
  // (128*56 + 256*224 = 64512). Each role sets its own limit at its entry.
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
    if (lane == 0) {
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % NS;
        if (!mbar_wait(&empty[s], ((it / NS) & 1) ^ 1, a_err, DEVERR_WAIT_PRODUCER)) break;
        uint8_t* sa_ = stage_base + s * C::kStage;
        uint8_t* sb_ = sa_ + C::kA;
        uint8_t* swp = sb_ + C::kB;
        if (it < nkb) {
          const int kb = kb_begin + it;
          mbar_arrive_expect_tx(&full[s], C::kB + C::kWP);
          tma_load_2d(sb_, &tm_xq, kb * kTileK, p0, &full[s]);
          bulk_load(swp, a.w_packed + (static_cast<size_t>(nt) * a.KB + kb) * kW4BlockBytes, C::kWP, &full[s]);
        } else {
          const int at = it - nkb;
          mbar_arrive_expect_tx(&full[s], C::kA + C::kB);
          tma_load_2d(sa_, &tm_bcat, at * kAdapterAtom, o0, &full[s]);
          tma_load_2d(sb_, &tm_ucat, at * kAdapterAtom, p0, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
    if (lane == 0) {
      const uint32_t id_i8 = idesc_i8(128, BN);
      const uint32_t id_ad = idesc_f16(128, BN);
      int gidx = 0;
      bool ok = true;
      for (int it = 0; it < n_iters && ok; ++it) {
        const int s = it % NS;
        const uint32_t ph = (it / NS) & 1;
        if (!mbar_wait(&full[s], ph, a_err, DEVERR_WAIT_MMA) || !mbar_wait(&afull[s], ph, a_err, DEVERR_WAIT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(stage_base + s * C::kStage);
        const uint32_t b_addr = a_addr + C::kA;
        if (it < nkb) {
          const int kb = kb_begin + it;
          for (int gi = 0; gi < gpb; ++gi) {
            const int gglob = kb * gpb + gi;
            if (gglob >= g_end) break;
            const int b = gidx & 1;
            if (!mbar_wait(&acce[b], ((gidx >> 1) & 1) ^ 1, a_err, DEVERR_WAIT_MMA)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d = tmem + b * BN;
            for (int kk = 0; kk < a.group / 32; ++kk) {
              const uint32_t koff = gi * a.group + kk * 32;
              mma_i8(d, smem_desc_sw128(a_addr + koff), smem_desc_sw128(b_addr + koff), id_i8, 1u);
            }
            tc_commit(&accf[b]);
            ++gidx;
          }
        } else {
          const int at = it - nkb;
          const int b = gidx & 1;
          if (at == 0) {
            if (!mbar_wait(&acce[b], ((gidx >> 1) & 1) ^ 1, a_err, DEVERR_WAIT_MMA)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          const uint32_t d = tmem + b * BN;
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(d, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32), id_ad,
                    (at > 0 || kk > 0) ? 1u : 0u);
          if (at == n_ad - 1) {
            tc_commit(&accf[b]);
            ++gidx;
          }
        }
        tc_commit(&empty[s]);
      }
      // make sure everything issued has completed before TMEM is released
      tc_commit(done);
      mbar_wait(done, 0, a_err, DEVERR_WAIT_TEARDOWN);
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ int4 -> int8 unpack
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
    const int u = threadIdx.x - 64;  // 0..63
    for (int it = 0; it < n_iters; ++it) {
      const int s = it % NS;
      if (!mbar_wait(&full[s], (it / NS) & 1, a_err, DEVERR_WAIT_UNPACK)) break;
      if (it < nkb) {
        uint8_t* sa_ = stage_base + s * C::kStage;
        const uint8_t* swp = sa_ + C::kA + C::kB;
#pragma unroll 2
        for (int i = 0; i < 8; ++i) {
          const int piece = u + 64 * i;  // 16-byte piece of the 8 KB block
          const int r = piece >> 2, q4 = piece & 3;
          const uint4 v = *reinterpret_cast<const uint4*>(swp + piece * 16);
          uint4 lo, hi;
          lo.x = sext_nibbles(v.x & 0x0F0F0F0Fu);
          lo.y = sext_nibbles(v.y & 0x0F0F0F0Fu);
          lo.z = sext_nibbles(v.z & 0x0F0F0F0Fu);
          lo.w = sext_nibbles(v.w & 0x0F0F0F0Fu);
          hi.x = sext_nibbles((v.x >> 4) & 0x0F0F0F0Fu);
          hi.y = sext_nibbles((v.y >> 4) & 0x0F0F0F0Fu);
          hi.z = sext_nibbles((v.z >> 4) & 0x0F0F0F0Fu);
          hi.w = sext_nibbles((v.w >> 4) & 0x0F0F0F0Fu);
          const int c_lo = 2 * q4, c_hi = 2 * q4 + 1;
          *reinterpret_cast<uint4*>(sa_ + r * 128 + ((c_lo ^ (r & 7)) << 4)) = lo;
          *reinterpret_cast<uint4*>(sa_ + r * 128 + ((c_hi ^ (r & 7)) << 4)) = hi;
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[s]);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 4..11)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
    const int q = warp & 3, h = (warp - 4) >> 2;
    const int o = o0 + 32 * q + lane;
    const bool o_ok = o < a.N;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    asm volatile("bar.sync 1, 256;" ::: "memory");  // sa_s / perm_s staged
    float acc[C::kCPT];
#pragma unroll
    for (int c = 0; c < C::kCPT; ++c) acc[c] = 0.0f;
    bool ok = true;
    int gidx = 0;
    float sw_next = (o_ok && n_groups > 0) ? __ldg(a.w_scale + static_cast<size_t>(g_begin) * a.N + o) : 0.0f;
    for (int g = 0; g < n_groups; ++g) {
      const int b = gidx & 1;
      const float sw = sw_next;
      if (g + 1 < n_groups && o_ok) sw_next = __ldg(a.w_scale + static_cast<size_t>(g_begin + g + 1) * a.N + o);
      if (!mbar_wait(&accf[b], (gidx >> 1) & 1, a_err, DEVERR_WAIT_EPILOGUE)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t base = tmem + lane_base + b * BN + h * C::kCPT;
#pragma unroll
      for (int c = 0; c < C::kCPT; c += C::kChunk) {
        uint32_t v[C::kChunk];
        tmem_ld<C::kChunk>(base + c, v);
        tmem_wait_ld();
        reg_fence(v);
        tmem_fill<C::kChunk>(base + c, kMagicBits);
        if (DBG && o_ok) {
#pragma unroll
          for (int i = 0; i < C::kChunk; ++i) {
            const int t = perm_s[h * C::kCPT + c + i];
            if (t >= 0)
              a.dbg_acc[(static_cast<size_t>(t) * a.N + o) * G_total + g_begin + g] =
                  static_cast<int32_t>(v[i] - kMagicBits);
          }
        }
#pragma unroll
        for (int i = 0; i < C::kChunk; ++i) acc[c + i] = fmaf(sw, __uint_as_float(v[i]) - kMagic, acc[c + i]);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[b]);
      ++gidx;
    }
    // per-token scale, adapters, store
#pragma unroll
    for (int c = 0; c < C::kCPT; ++c) acc[c] *= sa_s[h * C::kCPT + c];
    if (ok && n_ad > 0) {
      const int b = gidx & 1;
      if (mbar_wait(&accf[b], (gidx >> 1) & 1, a_err, DEVERR_WAIT_EPILOGUE)) {
        tc_fence_after();
        const uint32_t base = tmem + lane_base + b * BN + h * C::kCPT;
#pragma unroll
        for (int c = 0; c < C::kCPT; c += C::kChunk) {
          uint32_t v[C::kChunk];
          tmem_ld<C::kChunk>(base + c, v);
          tmem_wait_ld();
          reg_fence(v);
#pragma unroll
          for (int i = 0; i < C::kChunk; ++i) acc[c + i] = fmaf(su_s[h * C::kCPT + c + i], __uint_as_float(v[i]), acc[c + i]);
        }
      }
    }
    if (o_ok) {
      if (a.splits == 1) {
#pragma unroll
        for (int c = 0; c < C::kCPT; ++c) {
          const int t = perm_s[h * C::kCPT + c];
          if (t >= 0) {
            const size_t dst = static_cast<size_t>(t) * a.N + o;
            if (a.y_bf16) static_cast<uint16_t*>(a.Y)[dst] = f2bf(acc[c]);
            else static_cast<float*>(a.Y)[dst] = acc[c];
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < C::kCPT; ++c) {
          const int p = p0 + h * C::kCPT + c;
          if (p < a.T) a.partial[(static_cast<size_t>(split) * a.T + p) * a.N + o] = acc[c];
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------- U GEMM
// P[split][t][c] = sum over this split's K range of X[t][k] * A_catT[c][k].
// 192 threads: warp 0 TMA, warp 1 MMA (+ TMEM owner), warps 2-5 epilogue.
template <int NU>
struct UCfg {
  static constexpr int kA = 16384;     // 128 tokens x 64 bf16
  static constexpr int kB = NU * 128;  // NU adapter columns x 64 bf16
  static constexpr int kStage = kA + kB;
  static constexpr int kStages = 4;
  static constexpr int kTmemCols = NU <= 32 ? 32 : (NU <= 64 ? 64 : (NU <= 128 ? 128 : 256));
  static constexpr size_t kSmem = 1024 + size_t(kStages) * kStage + 256;
};

template <int NU>
__global__ void __launch_bounds__(192, 1)
    k_ugemm(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_acat, int T, int K,
            int R_pad, int kchunks_per_split, float* __restrict__ partial, int* a_err) {
  using C = UCfg<NU>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NS * C::kStage);
  uint64_t* full = bars;
  uint64_t* empty = bars + NS;
  uint64_t* accf = bars + 2 * NS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128, c0 = blockIdx.y * NU, split = blockIdx.z;
  const int nk_total = static_cast<int>(ceil_div(K, kAdapterAtom));
  const int kc_begin = split * kchunks_per_split;
  const int nk = max(0, min(nk_total, kc_begin + kchunks_per_split) - kc_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    mbar_fence_init();
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_acat);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      for (int it = 0; it < nk; ++it) {
        const int s = it % NS;
        if (!mbar_wait(&empty[s], ((it / NS) & 1) ^ 1, a_err, DEVERR_WAIT_PRODUCER)) break;
        uint8_t* sa_ = smem + s * C::kStage;
        mbar_arrive_expect_tx(&full[s], C::kStage);
        const int kx = (kc_begin + it) * kAdapterAtom;
        tma_load_2d(sa_, &tm_x, kx, m0, &full[s]);
        tma_load_2d(sa_ + C::kA, &tm_acat, kx, c0, &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id = idesc_bf16(128, NU);
      for (int it = 0; it < nk; ++it) {
        const int s = it % NS;
        if (!mbar_wait(&full[s], (it / NS) & 1, a_err, DEVERR_WAIT_MMA)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * C::kStage), b_addr = a_addr + C::kA;
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(tmem, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32), id,
                  (it > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      tc_commit(accf);
    }
  } else {
    const int q = warp & 3;
    const int row = m0 + 32 * q + lane;
    const bool ok = mbar_wait(accf, 0, a_err, DEVERR_WAIT_EPILOGUE);
    tc_fence_after();
    if (ok) {
      float* dst = partial + (static_cast<size_t>(split) * T + row) * R_pad + c0;
#pragma unroll 1
      for (int c = 0; c < NU; c += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + (static_cast<uint32_t>(32 * q) << 16) + c, v);
        tmem_wait_ld();
        reg_fence(v);
        if (row < T) {
          if (nk == 0) {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = 0u;
          }
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(dst + c + i) = make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                                                  __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int BN, bool DBG>
cudaError_t launch_qgemm_t(const CUtensorMap& tm_xq, const CUtensorMap& tm_bcat, const CUtensorMap& tm_ucat,
                           const QgemmArgs& a, cudaStream_t st) {
  using C = QCfg<BN>;
  // The epilogue warpgroups raise their register limit to 224 with setmaxnreg,
  // which waits until the producer warpgroup has released its share. That only
  // completes when the kernel was built with 168 registers per thread
  // (384 x 168 = 128 x 56 + 256 x 224), so refuse any other build.
  static int regs = -1;
  if (regs < 0) {
    cudaFuncAttributes fa;
    cudaError_t ea = cudaFuncGetAttributes(&fa, k_qgemm<BN, DBG>);
    if (ea != cudaSuccess) return ea;
    regs = fa.numRegs;
  }
  if (regs != 168) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(k_qgemm<BN, DBG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(ceil_div(a.N, kTileN)), static_cast<unsigned>(ceil_div(a.T, BN)),
            static_cast<unsigned>(a.splits));
  k_qgemm<BN, DBG><<<grid, 384, C::kSmem, st>>>(tm_xq, tm_bcat, tm_ucat, a);
  return cudaGetLastError();
}

template <int BN>
cudaError_t launch_qgemm_bn(const CUtensorMap& tm_xq, const CUtensorMap& tm_bcat, const CUtensorMap& tm_ucat,
                            const QgemmArgs& a, cudaStream_t st) {
  return a.dbg_acc ? launch_qgemm_t<BN, true>(tm_xq, tm_bcat, tm_ucat, a, st)
                   : launch_qgemm_t<BN, false>(tm_xq, tm_bcat, tm_ucat, a, st);
}

template <int NU>
cudaError_t launch_ugemm_t(const CUtensorMap& tm_x, const CUtensorMap& tm_acat, const UgemmPlan& p, int T, int K,
                           int R_pad, float* partial, int* err, cudaStream_t st) {
  using C = UCfg<NU>;
  cudaError_t e = cudaFuncSetAttribute(k_ugemm<NU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(ceil_div(T, 128)), static_cast<unsigned>(p.ntiles),
            static_cast<unsigned>(p.splits));
  k_ugemm<NU><<<grid, 192, C::kSmem, st>>>(tm_x, tm_acat, T, K, R_pad, p.kchunks_per_split, partial, err);
  return cudaGetLastError();
}

}  // namespace

int pick_qgemm_bn(int T, int N, int K, int* splits_out, int* kbps_out) {
  const int ntiles = static_cast<int>(ceil_div(N, kTileN));
  const int KB = static_cast<int>(ceil_div(K, kTileK));
  int bn;
  if (T <= 16) bn = 16;
  else if (T <= 32) bn = 32;
  else if (T <= 64) bn = 64;
  else if (T <= 128) bn = 128;
  else {
    // fill the 148 SMs: prefer 256-token tiles when they already give >= 1 full wave
    const int64_t tiles256 = int64_t(ntiles) * ceil_div(T, 256);
    bn = (tiles256 >= 148) ? 256 : 128;
  }
  const int64_t tiles = int64_t(ntiles) * ceil_div(T, bn);
  int splits = 1;
  if (tiles < 100 && KB >= 8) {
    splits = static_cast<int>(std::min<int64_t>(KB / 4, ceil_div(148, tiles)));
    if (splits < 1) splits = 1;
  }
  int kbps = static_cast<int>(ceil_div(KB, splits));
  splits = static_cast<int>(ceil_div(KB, kbps));
  *splits_out = splits;
  *kbps_out = kbps;
  return bn;
}

cudaError_t launch_qgemm(int BN, const CUtensorMap& tm_xq, const CUtensorMap& tm_bcat, const CUtensorMap& tm_ucat,
                         const QgemmArgs& a, cudaStream_t st) {
  switch (BN) {
    case 16: return launch_qgemm_bn<16>(tm_xq, tm_bcat, tm_ucat, a, st);
    case 32: return launch_qgemm_bn<32>(tm_xq, tm_bcat, tm_ucat, a, st);
    case 64: return launch_qgemm_bn<64>(tm_xq, tm_bcat, tm_ucat, a, st);
    case 128: return launch_qgemm_bn<128>(tm_xq, tm_bcat, tm_ucat, a, st);
    case 256: return launch_qgemm_bn<256>(tm_xq, tm_bcat, tm_ucat, a, st);
    default: return cudaErrorInvalidValue;
  }
}

UgemmPlan plan_ugemm(int T, int K, int R_pad) {
  UgemmPlan p;
  if (R_pad <= 256) p.nu = R_pad;
  else if (R_pad % 256 == 0) p.nu = 256;
  else if (R_pad % 192 == 0) p.nu = 192;
  else if (R_pad % 128 == 0) p.nu = 128;
  else p.nu = 64;
  p.ntiles = static_cast<int>(ceil_div(R_pad, p.nu));
  const int mtiles = static_cast<int>(ceil_div(T, 128));
  const int nk = static_cast<int>(ceil_div(K, kAdapterAtom));
  int splits = static_cast<int>(ceil_div(2 * 148, int64_t(mtiles) * p.ntiles));
  splits = std::max(1, std::min(splits, std::max(1, nk / 2)));
  p.kchunks_per_split = static_cast<int>(ceil_div(nk, splits));
  p.splits = static_cast<int>(ceil_div(nk, p.kchunks_per_split));
  return p;
}

cudaError_t launch_ugemm(const CUtensorMap& tm_x, const CUtensorMap& tm_acat, const UgemmPlan& plan, int T, int K,
                         int R_pad, float* partial, int* err, cudaStream_t st) {
  switch (plan.nu) {
    case 64: return launch_ugemm_t<64>(tm_x, tm_acat, plan, T, K, R_pad, partial, err, st);
    case 128: return launch_ugemm_t<128>(tm_x, tm_acat, plan, T, K, R_pad, partial, err, st);
    case 192: return launch_ugemm_t<192>(tm_x, tm_acat, plan, T, K, R_pad, partial, err, st);
    case 256: return launch_ugemm_t<256>(tm_x, tm_acat, plan, T, K, R_pad, partial, err, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qe
