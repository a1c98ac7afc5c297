// Tensor-core kernels (tcgen05 + TMEM + TMA) of the QE linear layer.
//
// k_qgemm: the main W4 x A8/A6 product with the QE epilogue. The tile is
//   M = 128 output channels (weights are the A operand, so each TMEM lane is
//   one output row) by N = BN token positions in bucket order (the B
//   operand). Each pipeline stage covers 128 input channels:
//     warp 0      TMA producer: activation codes (tensor map, 128B swizzle),
//                 plus one bulk copy of the 8 KB packed-int4 weight block
//     warps 12-15 unpack the int4 block into int8 in the 128B-swizzled A layout
//     warps 1-2   one thread each issues tcgen05.mma kind::i8 for alternate
//                 stages, one TMEM accumulator buffer per quantization group
//                 (2 buffers at BN >= 192, 4 below, so the MMA runs ahead of the
//                 epilogue; each issuer owns half of them)
//     warps 4-11  epilogue: the per-group promotion acc += sw[o,j] * float(int32)
//                 in registers (f32x2, the next TMEM chunk loading meanwhile),
//                 then * sa[t], + adapter MMA result, and a scatter of the row
//                 to token order
//   The kernel is persistent: one CTA per SM walks a static list of
//   (output tile, token tile, K split) units, so barriers and TMEM are set up
//   once and the next unit's loads and MMAs overlap the last unit's stores.
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
#include <utility>

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
  static constexpr int kA = 16384;                 // 128 rows x 128 B (int8 K=128 or fp16 K=64)
  static constexpr int kB = BN * 128;
  static constexpr int kWP = kW4BlockBytes;         // packed int4 block
  static constexpr int kStage = kA + kB + kWP;
  static constexpr int kStages = (BN >= 192) ? 3 : (BN >= 128 ? 4 : (BN >= 64 ? 5 : 6));
  static constexpr int kNBuf = (BN >= 192) ? 2 : 4;  // TMEM accumulator buffers
  static_assert(kNBuf % 2 == 0, "each MMA issuer owns half of the buffers");
  // TMEM is allocated in powers of two (>= 32 columns)
  static constexpr int kTmemCols = (kNBuf * BN <= 32) ? 32 : (kNBuf * BN <= 128 ? 128 : (kNBuf * BN <= 256 ? 256 : 512));
  static constexpr int kCPT = BN / 2;              // columns per epilogue thread
  static constexpr int kChunk = (kCPT >= 96) ? 16 : ((kCPT >= 32) ? 32 : kCPT);
  static constexpr int kNChunk = kCPT / kChunk;
  static constexpr int kOut = 32768;               // output staging (two 16 KB halves, one per epilogue warpgroup)
  static constexpr size_t kSmem = 1024 /*align slack*/ + size_t(kStages) * kStage + kOut + 1024 /*barriers etc*/ +
                                  size_t(BN) * 12 /*sa + su + perm*/;
  // setmaxnreg split of the 512 x 128 launch registers: the producer/MMA warpgroup and the
  // unpack warpgroup drop to kRegLow, the two epilogue warpgroups rise to kRegHigh
  // (256 * kRegLow + 256 * kRegHigh = 65536); the values were picked per tile width by spill counts.
  static constexpr int kRegLow = (BN >= 128) ? 72 : 56;
  static constexpr int kRegHigh = (65536 - 256 * kRegLow) / 256;
  static_assert(256 * kRegLow + 256 * kRegHigh == 65536 && kRegLow % 8 == 0 && kRegHigh % 8 == 0, "register split");
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

// acc[i..i+1] += sw * (float(v[i..i+1]) - 1.5*2^23), two lanes per instruction (f32x2).
// The subtraction is exact (both operands lie in [2^23, 2^24)); the FMA rounds once.
__device__ __forceinline__ void promote2(float& a0, float& a1, uint32_t v0, uint32_t v1, uint64_t sw2,
                                         uint64_t magic2) {
  uint64_t x, acc;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "r"(v0), "r"(v1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(acc) : "f"(a0), "f"(a1));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(x) : "l"(x), "l"(magic2));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(acc) : "l"(x), "l"(sw2), "l"(acc));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(acc));
}

__device__ __forceinline__ uint64_t pack2(float x) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(x));
  return r;
}

// One unit of work: a 128-row output tile, a BN-position token tile and a K split.
struct Unit {
  int nt, p0, split, kb_begin, nkb, n_ad, g_begin, n_groups;
};

__device__ __forceinline__ Unit make_unit(const QgemmArgs& a, int BN, int u) {
  Unit w;
  const int NT = static_cast<int>(ceil_div(a.N, kTileN));
  const int PT = static_cast<int>(ceil_div(a.T, BN));
  w.nt = u % NT;
  const int rest = u / NT;
  w.p0 = (rest % PT) * BN;
  w.split = rest / PT;
  w.kb_begin = w.split * a.kb_per_split;
  const int kb_end = min(a.KB, w.kb_begin + a.kb_per_split);
  w.nkb = max(0, kb_end - w.kb_begin);
  w.n_ad = (w.split == 0) ? a.adapter_atoms : 0;
  const int gpb = kTileK / a.group;
  const int G_total = a.K / a.group;
  w.g_begin = w.kb_begin * gpb;
  w.n_groups = max(0, min(G_total, kb_end * gpb) - w.g_begin);
  return w;
}


// Largest divisor of cpt that is at most cap (the columns one staging pass can hold).
__host__ __device__ constexpr int pass_columns(int cpt, int cap) {
  int d = cap < cpt ? cap : cpt;
  while (cpt % d != 0) --d;
  return d;
}

// Writes one epilogue warpgroup's half tile (128 output channels x CPT token columns) to Y.
// Each pass moves PC columns: every thread puts its values for those columns into the
// warpgroup's 16 KB staging buffer (column-major by token), then the 128 threads copy
// whole row segments (128 channels = 256 B bf16 / 512 B fp32) to Y[token] with 16-byte
// stores. Rows go to perm[p] (token order), or to position p of this split's partial
// buffer. Every thread runs every pass and barrier, whatever `ok` is.
template <int CPT, int ELEM>
__device__ __forceinline__ void store_tile(const float (&acc)[CPT], uint8_t* stage, const int32_t* perm_cols,
                                           const Unit& w, const QgemmArgs& a, int o0, int o_local, int wt, int h,
                                           bool ok, bool to_partial) {
  constexpr int kRowBytes = 128 * ELEM;
  constexpr int kPC = pass_columns(CPT, 16384 / kRowBytes);  // columns per pass (divides CPT)
  constexpr int kChunksPerRow = kRowBytes / 16;
  constexpr int kElemsPerChunk = 16 / ELEM;
  const bool vec_ok = ((static_cast<size_t>(a.N) * ELEM) % 16) == 0;
#pragma unroll
  for (int pass = 0; pass < CPT / kPC; ++pass) {
#pragma unroll
    for (int c = 0; c < kPC; ++c) {
      const float v = acc[pass * kPC + c];
      if constexpr (ELEM == 2) {
        *reinterpret_cast<uint16_t*>(stage + c * kRowBytes + o_local * 2) = f2bf(v);
      } else {
        *reinterpret_cast<float*>(stage + c * kRowBytes + o_local * 4) = v;
      }
    }
    asm volatile("bar.sync %0, 128;" ::"r"(2 + h) : "memory");
    if (ok) {
#pragma unroll
      for (int k = 0; k < (kPC * kChunksPerRow) / 128; ++k) {
        const int ch = wt + 128 * k;
        const int c = ch / kChunksPerRow, part = ch % kChunksPerRow;
        const int col = pass * kPC + c;  // column inside this warpgroup's half
        const int p = w.p0 + h * CPT + col;
        const int row = to_partial ? (p < a.T ? p : -1) : perm_cols[col];
        if (row < 0) continue;
        const int of = o0 + part * kElemsPerChunk;
        if (of >= a.N) continue;
        uint8_t* dst_base = to_partial
                                ? reinterpret_cast<uint8_t*>(a.partial + (static_cast<size_t>(w.split) * a.T + row) * a.N)
                                : static_cast<uint8_t*>(a.Y) + static_cast<size_t>(row) * a.N * ELEM;
        const uint8_t* src = stage + c * kRowBytes + part * 16;
        if (vec_ok && of + kElemsPerChunk <= a.N) {
          *reinterpret_cast<uint4*>(dst_base + static_cast<size_t>(of) * ELEM) = *reinterpret_cast<const uint4*>(src);
        } else {
          for (int e = 0; e < kElemsPerChunk && of + e < a.N; ++e) {
            if constexpr (ELEM == 2)
              *reinterpret_cast<uint16_t*>(dst_base + static_cast<size_t>(of + e) * 2) =
                  *reinterpret_cast<const uint16_t*>(src + e * 2);
            else
              *reinterpret_cast<float*>(dst_base + static_cast<size_t>(of + e) * 4) =
                  *reinterpret_cast<const float*>(src + e * 4);
          }
        }
      }
    }
    asm volatile("bar.sync %0, 128;" ::"r"(2 + h) : "memory");
  }
}

template <int BN, bool DBG>
__global__ void __launch_bounds__(512, 1)
    k_qgemm(const __grid_constant__ CUtensorMap tm_xq, const __grid_constant__ CUtensorMap tm_bcat,
            const __grid_constant__ CUtensorMap tm_ucat, const QgemmArgs a) {
  using C = QCfg<BN>;
  constexpr int NS = C::kStages;
  constexpr int NB = C::kNBuf;
  int* const a_err = a.err;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* out_stage = smem + NS * C::kStage;  // [2][16 KB] output transpose buffers
  uint64_t* bars = reinterpret_cast<uint64_t*>(out_stage + C::kOut);
  uint64_t* full = bars;            // [NS] TMA bytes landed
  uint64_t* afull = bars + NS;      // [NS] unpack done (4 warp arrivals)
  uint64_t* empty = bars + 2 * NS;  // [NS] MMAs done reading the stage
  uint64_t* accf = bars + 3 * NS;   // [NB] accumulator buffer ready for the epilogue
  uint64_t* acce = accf + NB;       // [NB] accumulator buffer drained and re-biased (8 warp arrivals)
  uint64_t* done = acce + NB;       // [1] teardown
  uint64_t* adone = done + 1;       // [1] adapter block: its issuer waited for all of its stages
  uint64_t* aack = adone + 1;       // [1] adapter block: the other issuer saw adone
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(aack + 1);
  float* sa_s = reinterpret_cast<float*>(out_stage + C::kOut + 512);
  float* su_s = sa_s + BN;
  int32_t* perm_s = reinterpret_cast<int32_t*>(su_s + BN);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NT = static_cast<int>(ceil_div(a.N, kTileN));
  const int PT = static_cast<int>(ceil_div(a.T, BN));
  const int n_units = NT * PT * a.splits;
  const int gpb = kTileK / a.group;  // groups per 128-channel block
  const int G_total = a.K / a.group;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&afull[s], 4);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 8);
    }
    mbar_init(done, 2);
    mbar_init(adone, 1);
    mbar_init(aack, 1);
    mbar_arrive(aack);  // phase 0: nothing to acknowledge before the first adapter block
    mbar_fence_init();
    prefetch_tmap(&tm_xq);
    if (a.adapter_atoms) {
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

  if (warp >= 4 && warp < 12) {
    // epilogue threads put the magic bias into every accumulator buffer once
    const int q = warp & 3, h = (warp - 4) >> 2;
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int c = 0; c < C::kCPT; c += C::kChunk)
        tmem_fill<C::kChunk>(tmem + (static_cast<uint32_t>(32 * q) << 16) + b * BN + h * C::kCPT + c, kMagicBits);
    tmem_wait_st();
    tc_fence_before();
  }
  __syncthreads();
  // everything above touched only this CTA's shared memory and TMEM
  grid_dep_wait();
  grid_dep_launch();

  // Roles: warp 0 TMA producer, warps 1-2 MMA issuers (warp 3 idle), warps 4-11 epilogue,
  // warps 12-15 unpack. Register split: 256 * kRegLow + 256 * kRegHigh = 512 x 128 launch
  // registers; each role sets its own limit at its entry.
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kRegLow) : "memory");
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const Unit w = make_unit(a, BN, u);
        for (int i = 0; i < w.nkb + w.n_ad; ++i, ++it) {
          const int s = it % NS;
          if (!mbar_wait(&empty[s], ((it / NS) & 1) ^ 1, a_err, DEVERR_WAIT_PRODUCER)) {
            ok = false;
            break;
          }
          uint8_t* sa_ = stage_base + s * C::kStage;
          uint8_t* sb_ = sa_ + C::kA;
          uint8_t* swp = sb_ + C::kB;
          if (i < w.nkb) {
            const int kb = w.kb_begin + i;
            mbar_arrive_expect_tx(&full[s], C::kB + C::kWP);
            tma_load_2d(sb_, &tm_xq, kb * kTileK, w.p0, &full[s]);
            bulk_load(swp, a.w_packed + (static_cast<size_t>(w.nt) * a.KB + kb) * kW4BlockBytes, C::kWP, &full[s]);
          } else {
            const int at = i - w.nkb;
            mbar_arrive_expect_tx(&full[s], C::kA + C::kB);
            tma_load_2d(sa_, &tm_bcat, at * kAdapterAtom, w.nt * kTileN, &full[s]);
            tma_load_2d(sb_, &tm_ucat, at * kAdapterAtom, w.p0, &full[s]);
          }
        }
      }
      drain_ring(full, NS, it);
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    // One thread issuing every tcgen05.mma cannot keep the tensor pipe busy: each issue,
    // barrier wait and commit costs it tens of cycles. Two issuers split the stages by
    // parity of the running stage index. A unit's adapter atoms accumulate into one TMEM
    // buffer, so one issuer takes all of them and their fp32 sums keep a fixed order.
    // The unpack warps wait for the TMA bytes before they arrive on afull, so afull alone
    // tells an issuer that both operands of the stage are in shared memory.
    // A parity wait is only sound when the waiter is at most one phase ahead of the barrier.
    // An issuer skips the other's stages, so two rules keep it within one phase:
    //  - TMEM buffers are owned: issuer q uses buffers q, q+2, ... in turn, so its waits on
    //    a buffer's acce are for consecutive drains of that buffer;
    //  - after skipping another issuer's adapter block (possibly longer than the stage ring),
    //    an issuer waits on adone, which the owner arrives on once it has waited for every
    //    stage of the block; the owner of the next block first waits on aack, so adone is
    //    never two blocks ahead of its waiter.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kRegLow) : "memory");
    const int qi = warp - 1;
    if (lane == 0) {
      const uint32_t id_i8 = idesc_i8(128, BN);
      const uint32_t id_ad = idesc_f16(128, BN);
      // Descriptors are built once; a stage or a 32-byte K step only moves the start address
      // field (16-byte units in the low bits, no carry below 256 KB of shared memory).
      const uint64_t desc0 = smem_desc_sw128(smem_u32(stage_base));
      constexpr int kOwn = NB / 2;  // TMEM buffers per issuer
      int it = 0;
      uint32_t own = 0, ablk = 0;  // groups this issuer took (mod 8), adapter blocks seen (mod 2)
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const Unit w = make_unit(a, BN, u);
        const int ad_owner = (it + w.nkb) & 1;
        for (int i = 0; i < w.nkb + w.n_ad && ok; ++i, ++it) {
          const int s = it % NS;
          const uint32_t ph = (it / NS) & 1;
          const uint64_t da = desc0 + static_cast<uint64_t>((s * C::kStage) >> 4);
          const uint64_t db = da + (C::kA >> 4);
          if (i < w.nkb) {
            if ((it & 1) != qi) continue;
            const int kb = w.kb_begin + i;
            const int ng = max(0, min(gpb, w.g_begin + w.n_groups - kb * gpb));
            if (!mbar_wait(&afull[s], ph, a_err, DEVERR_WAIT_MMA)) {
              ok = false;
              break;
            }
            // four K steps of 32 per stage: one group (g = 128) or two (g = 64)
#pragma unroll
            for (int gi = 0; gi < 2; ++gi) {
              if (gi >= ng) break;
              const int b = qi + 2 * static_cast<int>(own % kOwn);
              const uint32_t use = own / kOwn;
              own = (own + 1) & 7u;
              if (!mbar_wait(&acce[b], (use & 1) ^ 1, a_err, DEVERR_WAIT_MMA)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t d = tmem + b * BN;
              if (gpb == 1) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) mma_i8(d, da + 2 * kk, db + 2 * kk, id_i8, 1u);
              } else {
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) mma_i8(d, da + 4 * gi + 2 * kk, db + 4 * gi + 2 * kk, id_i8, 1u);
              }
              tc_commit(&accf[b]);
            }
          } else {
            const int at = i - w.nkb;
            if (ad_owner != qi) {
              if (at == w.n_ad - 1) {
                if (!mbar_wait(adone, ablk, a_err, DEVERR_WAIT_MMA)) {
                  ok = false;
                  break;
                }
                mbar_arrive(aack);
                ablk ^= 1u;
              }
              continue;
            }
            const int b = qi + 2 * static_cast<int>(own % kOwn);
            if (!mbar_wait(&afull[s], ph, a_err, DEVERR_WAIT_MMA)) {
              ok = false;
              break;
            }
            if (at == 0) {
              if (!mbar_wait(&acce[b], ((own / kOwn) & 1u) ^ 1u, a_err, DEVERR_WAIT_MMA)) {
                ok = false;
                break;
              }
            }
            tc_fence_after();
            const uint32_t d = tmem + b * BN;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) mma_f16(d, da + 2 * kk, db + 2 * kk, id_ad, (at > 0 || kk > 0) ? 1u : 0u);
            if (at == w.n_ad - 1) {
              tc_commit(&accf[b]);
              own = (own + 1) & 7u;
            }
          }
          tc_commit(&empty[s]);
          if (i >= w.nkb && i - w.nkb == w.n_ad - 1) {
            // this issuer owned the adapter block and has waited for all of its stages
            if (!mbar_wait(aack, ablk, a_err, DEVERR_WAIT_MMA)) {
              ok = false;
              break;
            }
            mbar_arrive(adone);
            ablk ^= 1u;
          }
        }
      }
      // make sure everything this thread issued has completed before TMEM is released
      tc_commit(done);
      mbar_wait(done, 0, a_err, DEVERR_WAIT_TEARDOWN);
    }
  } else if (warp == 3) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kRegLow) : "memory");
  } else if (warp >= 12) {
    // ------------------------------------------------------------ int4 -> int8 unpack (warps 12..15)
    // Each code goes to the high nibble of its byte, so the byte reads as the int8 16*q.
    // The factor 16 is folded into the group scale (sw/16, exact), and |16*acc| stays below 2^22.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kRegLow) : "memory");
    const int uth = threadIdx.x - 384;  // 0..127
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const Unit w = make_unit(a, BN, u);
      for (int i = 0; i < w.nkb + w.n_ad; ++i, ++it) {
        const int s = it % NS;
        if (!mbar_wait(&full[s], (it / NS) & 1, a_err, DEVERR_WAIT_UNPACK)) {
          ok = false;
          break;
        }
        if (i < w.nkb) {
          uint8_t* sa_ = stage_base + s * C::kStage;
          const uint8_t* swp = sa_ + C::kA + C::kB;
          uint4 v[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const uint4*>(swp + (uth + 128 * j) * 16);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int piece = uth + 128 * j;  // 16-byte piece of the 8 KB block
            const int r = piece >> 2, q4 = piece & 3;
            uint4 lo, hi;
            lo.x = (v[j].x << 4) & 0xF0F0F0F0u;
            lo.y = (v[j].y << 4) & 0xF0F0F0F0u;
            lo.z = (v[j].z << 4) & 0xF0F0F0F0u;
            lo.w = (v[j].w << 4) & 0xF0F0F0F0u;
            hi.x = v[j].x & 0xF0F0F0F0u;
            hi.y = v[j].y & 0xF0F0F0F0u;
            hi.z = v[j].z & 0xF0F0F0F0u;
            hi.w = v[j].w & 0xF0F0F0F0u;
            const int c_lo = 2 * q4, c_hi = 2 * q4 + 1;
            *reinterpret_cast<uint4*>(sa_ + r * 128 + ((c_lo ^ (r & 7)) << 4)) = lo;
            *reinterpret_cast<uint4*>(sa_ + r * 128 + ((c_hi ^ (r & 7)) << 4)) = hi;
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[s]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 4..11)
    // Control flow here depends only on the unit schedule, never on a wait's
    // outcome: the named barriers below must be reached by every epilogue warp.
    // After a wait runs out, `ok` (warp-uniform) turns every later wait and TMEM access off.
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::kRegHigh) : "memory");
    const int q = warp & 3, h = (warp - 4) >> 2;
    const int et = threadIdx.x - 128;      // 0..255
    const int wt = et & 127;               // thread index inside this epilogue warpgroup
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const uint64_t magic2 = pack2(kMagic);
    uint8_t* my_out = out_stage + h * (C::kOut / 2);
    // group -> TMEM buffer as the issuers assign it: K block i of a unit is issued by the
    // issuer of the stage's parity, which takes its buffers q, q+2, ... in turn
    constexpr int kOwn = NB / 2;
    uint32_t bstate = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
      const Unit w = make_unit(a, BN, u);
      const int o0 = w.nt * kTileN;
      const int o = o0 + 32 * q + lane;
      const bool o_ok = o < a.N;
      // this unit's per-position scales and token ids: copied asynchronously into shared memory
      // (after everyone finished the previous unit's store), waited for when the epilogue needs them
      asm volatile("bar.sync 1, 256;" ::: "memory");
      for (int c = et; c < BN; c += 256) {
        const int p = w.p0 + c;
        if (p < a.T) {
          cp_async4(&sa_s[c], a.sa_sorted + p);
          if (a.su_sorted) cp_async4(&su_s[c], a.su_sorted + p);
          else su_s[c] = 0.0f;
          cp_async4(&perm_s[c], a.perm + p);
        } else {
          sa_s[c] = 0.0f;
          su_s[c] = 0.0f;
          perm_s[c] = -1;
        }
      }
      cp_async_commit();
      if (DBG) {
        cp_async_wait_all();
        asm volatile("bar.sync 1, 256;" ::: "memory");
      }
      float acc[C::kCPT];
#pragma unroll
      for (int c = 0; c < C::kCPT; ++c) acc[c] = 0.0f;
      // weight codes enter the MMA as 16*q, so the group scale is applied as sw/16 (exact).
      // The scales are loaded kSwAhead groups ahead (a load can outlast a group's drain).
      constexpr int kSwAhead = 2;
      const size_t sw0 = static_cast<size_t>(w.g_begin) * a.N + o;  // scale of (o, first group)
      float swq[kSwAhead];
#pragma unroll
      for (int j = 0; j < kSwAhead; ++j)
        swq[j] = (o_ok && j < w.n_groups) ? load_scale(a.w_scale, sw0 + static_cast<size_t>(j) * a.N, a.sw_f16) : 0.0f;
      for (int g = 0; g < w.n_groups; ++g) {
        uint32_t use;
        const int b = epi_next_buffer<kOwn>(bstate, static_cast<int>(bstate & 1u), use);
        // bit 0 follows the stage parity: flip it after the last group of each K block
        if (a.group == kTileK || (g & 1) || g + 1 == w.n_groups) bstate ^= 1u;
        const uint64_t sw2 = pack2(swq[0] * 0.0625f);
#pragma unroll
        for (int j = 0; j + 1 < kSwAhead; ++j) swq[j] = swq[j + 1];
        swq[kSwAhead - 1] = (o_ok && g + kSwAhead < w.n_groups)
                                ? load_scale(a.w_scale, sw0 + static_cast<size_t>(g + kSwAhead) * a.N, a.sw_f16)
                                : 0.0f;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&accf[b], use & 1, a_err, DEVERR_WAIT_EPILOGUE));
        if (!ok) continue;
        tc_fence_after();
        const uint32_t base = tmem + lane_base + b * BN + h * C::kCPT;
        // chunk c+1 loads while chunk c is promoted; each drained chunk is re-biased at once
        uint32_t va[C::kChunk], vb[C::kChunk];
        tmem_ld<C::kChunk>(base, va);
        tmem_wait_ld();
        reg_fence(va);
#pragma unroll
        for (int c = 0; c < C::kNChunk; ++c) {
          uint32_t(&cur)[C::kChunk] = (c & 1) ? vb : va;
          uint32_t(&nxt)[C::kChunk] = (c & 1) ? va : vb;
          if (c + 1 < C::kNChunk) tmem_ld<C::kChunk>(base + (c + 1) * C::kChunk, nxt);
          tmem_fill<C::kChunk>(base + c * C::kChunk, kMagicBits);
          if (DBG && o_ok) {
#pragma unroll
            for (int i = 0; i < C::kChunk; ++i) {
              const int t = perm_s[h * C::kCPT + c * C::kChunk + i];
              if (t >= 0)
                a.dbg_acc[(static_cast<size_t>(t) * a.N + o) * G_total + w.g_begin + g] =
                    static_cast<int32_t>(cur[i] - kMagicBits) / 16;
            }
          }
#pragma unroll
          for (int i = 0; i < C::kChunk; i += 2)
            promote2(acc[c * C::kChunk + i], acc[c * C::kChunk + i + 1], cur[i], cur[i + 1], sw2, magic2);
          if (c + 1 < C::kNChunk) {
            tmem_wait_ld();
            reg_fence(nxt);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[b]);
      }
      cp_async_wait_all();
      asm volatile("bar.sync 1, 256;" ::: "memory");
      // per-token scale
      const float4* sa4 = reinterpret_cast<const float4*>(sa_s + h * C::kCPT);
#pragma unroll
      for (int c = 0; c < C::kCPT; c += 4) {
        const float4 f = sa4[c / 4];
        acc[c] *= f.x;
        acc[c + 1] *= f.y;
        acc[c + 2] *= f.z;
        acc[c + 3] *= f.w;
      }
      // adapters: acc += su[t] * (U_cat . B_cat^T)
      if (w.n_ad > 0) {
        uint32_t use;
        const int b = epi_next_buffer<kOwn>(bstate, static_cast<int>(bstate & 1u), use);
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&accf[b], use & 1, a_err, DEVERR_WAIT_EPILOGUE));
        if (ok) {
          tc_fence_after();
          const uint32_t base = tmem + lane_base + b * BN + h * C::kCPT;
          const float4* su4 = reinterpret_cast<const float4*>(su_s + h * C::kCPT);
#pragma unroll
          for (int c = 0; c < C::kCPT; c += C::kChunk) {
            uint32_t v[C::kChunk];
            tmem_ld<C::kChunk>(base + c, v);
            tmem_wait_ld();
            reg_fence(v);
            tmem_fill<C::kChunk>(base + c, kMagicBits);
#pragma unroll
            for (int i = 0; i < C::kChunk; i += 4) {
              const float4 f = su4[(c + i) / 4];
              acc[c + i] = fmaf(f.x, __uint_as_float(v[i]), acc[c + i]);
              acc[c + i + 1] = fmaf(f.y, __uint_as_float(v[i + 1]), acc[c + i + 1]);
              acc[c + i + 2] = fmaf(f.z, __uint_as_float(v[i + 2]), acc[c + i + 2]);
              acc[c + i + 3] = fmaf(f.w, __uint_as_float(v[i + 3]), acc[c + i + 3]);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acce[b]);
        }
      }
      // store: transpose through shared memory, then write whole row segments with 16-byte stores
      if (a.splits == 1 && a.y_bf16) store_tile<C::kCPT, 2>(acc, my_out, perm_s + h * C::kCPT, w, a, o0, 32 * q + lane, wt, h, ok, false);
      else store_tile<C::kCPT, 4>(acc, my_out, perm_s + h * C::kCPT, w, a, o0, 32 * q + lane, wt, h, ok, a.splits > 1);
      bstate ^= static_cast<uint32_t>(w.n_ad) & 1u;
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
// P[slot][t][c] = sum over this split's K range of X[t][k] * A_catT[c][k] for c in this CTA's
// column tile: the adapter down-projections and the router logits in one bf16 tcgen05 GEMM
// (M = 128 tokens, N = adapter + router columns, K split across CTAs, fp32 partial slots).
// 192 threads: warp 0 TMA, warp 1 MMA (+ TMEM owner), warps 2-5 epilogue.
template <int NU>
struct UCfg {
  static constexpr int kA = 16384;     // 128 tokens x 64 bf16
  static constexpr int kB = NU * 128;  // NU columns x 64 bf16
  static constexpr int kStage = kA + kB;
  static constexpr int kStages = 4;
  static constexpr int kTmemCols = NU <= 32 ? 32 : (NU <= 64 ? 64 : (NU <= 128 ? 128 : 256));
  static constexpr size_t kSmem = 1024 + size_t(kStages) * kStage + 256;
};

template <int NU>
__global__ void __launch_bounds__(192, 1)
    k_ugemm(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_acat, int T, int K,
            int R_tot, int kchunks_per_split, float* __restrict__ partial, unsigned* zero_ctr, int* a_err) {
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
  grid_dep_wait();
  grid_dep_launch();
  if (zero_ctr && threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) *zero_ctr = 0u;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      for (; it < nk; ++it) {
        const int s = it % NS;
        if (!mbar_wait(&empty[s], ((it / NS) & 1) ^ 1, a_err, DEVERR_WAIT_PRODUCER)) break;
        uint8_t* sa_ = smem + s * C::kStage;
        const int kx = (kc_begin + it) * kAdapterAtom;
        mbar_arrive_expect_tx(&full[s], C::kA + C::kB);
        tma_load_2d(sa_, &tm_x, kx, m0, &full[s]);
        tma_load_2d(sa_ + C::kA, &tm_acat, kx, c0, &full[s]);
      }
      drain_ring(full, NS, it);
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
    const int r = 32 * q + lane;  // tile row == TMEM lane of this thread
    const int row = m0 + r;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(accf, 0, a_err, DEVERR_WAIT_EPILOGUE));
    tc_fence_after();
    if (ok) {
      float* dst = partial + (static_cast<size_t>(split) * T + row) * R_tot + c0;
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

// Launch with programmatic stream serialization: the kernel may be scheduled while the previous
// kernel on the stream drains, and waits for it (grid_dep_wait) after its own set-up.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int BN, bool DBG>
cudaError_t launch_qgemm_t(const CUtensorMap& tm_xq, const CUtensorMap& tm_bcat, const CUtensorMap& tm_ucat,
                           const QgemmArgs& a, cudaStream_t st) {
  using C = QCfg<BN>;
  // The epilogue warpgroups raise their register limit with setmaxnreg,
  // which waits until the other warpgroups have released their share. That only
  // completes when the kernel was built with 128 registers per thread
  // (512 x 128 = 256 x kRegLow + 256 x kRegHigh), so refuse any other build.
  static int regs = -1;
  if (regs < 0) {
    cudaFuncAttributes fa;
    cudaError_t ea = cudaFuncGetAttributes(&fa, k_qgemm<BN, DBG>);
    if (ea != cudaSuccess) return ea;
    regs = fa.numRegs;
  }
  if (regs != 128) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(k_qgemm<BN, DBG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM (or per unit when there are fewer units), each loops over units
  static int n_sm = 0;
  if (n_sm == 0) {
    int dev = 0;
    cudaError_t ed = cudaGetDevice(&dev);
    if (ed == cudaSuccess) ed = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (ed != cudaSuccess) return ed;
  }
  const int64_t units = ceil_div(a.N, kTileN) * ceil_div(a.T, BN) * a.splits;
  const unsigned grid = static_cast<unsigned>(units < n_sm ? units : n_sm);
  return launch_pdl(k_qgemm<BN, DBG>, dim3(grid), dim3(512), C::kSmem, st, tm_xq, tm_bcat, tm_ucat, a);
}

template <int BN>
cudaError_t launch_qgemm_bn(const CUtensorMap& tm_xq, const CUtensorMap& tm_bcat, const CUtensorMap& tm_ucat,
                            const QgemmArgs& a, cudaStream_t st) {
  return a.dbg_acc ? launch_qgemm_t<BN, true>(tm_xq, tm_bcat, tm_ucat, a, st)
                   : launch_qgemm_t<BN, false>(tm_xq, tm_bcat, tm_ucat, a, st);
}

template <int NU>
cudaError_t launch_ugemm_t(const CUtensorMap& tm_x, const CUtensorMap& tm_acat, const UgemmPlan& p, int T, int K,
                           int R_tot, float* partial, unsigned* zero_ctr, int* err, cudaStream_t st) {
  using C = UCfg<NU>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k_ugemm<NU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(C::kSmem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid(static_cast<unsigned>(ceil_div(T, 128)), static_cast<unsigned>(p.ntiles),
            static_cast<unsigned>(p.splits));
  return launch_pdl(k_ugemm<NU>, grid, dim3(192), C::kSmem, st, tm_x, tm_acat, T, K, R_tot, p.kchunks_per_split,
                    partial, zero_ctr, err);
}

}  // namespace

// Token-tile width and K split of the int8 GEMM. Small T takes the smallest tile that covers it.
// Otherwise each candidate width is priced by a model of the persistent kernel: rounds of units
// over the SMs, each unit costing its groups at the width's measured per-group time plus a fixed
// unit cost (epilogue scaling, adapter and store). Wider tiles run the tensor core closer to its
// peak, narrower ones fill the SMs better.
int pick_qgemm_bn(int T, int N, int K, int* splits_out, int* kbps_out) {
  const int ntiles = static_cast<int>(ceil_div(N, kTileN));
  const int KB = static_cast<int>(ceil_div(K, kTileK));
  int bn;
  if (T <= 16) bn = 16;
  else if (T <= 32) bn = 32;
  else if (T <= 64) bn = 64;
  else if (T <= 128) bn = 128;
  else {
    constexpr int kCand[3] = {128, 192, 256};
    constexpr double kGroupUs[3] = {0.37, 0.46, 0.56};  // per 128-deep K block
    constexpr double kUnitUs = 4.0;
    double best = 1e30;
    bn = 128;
    for (int i = 0; i < 3; ++i) {
      const int64_t units = int64_t(ntiles) * ceil_div(T, kCand[i]);
      const int64_t rounds = ceil_div(units, 148);
      const double cost = double(rounds) * (KB * kGroupUs[i] + kUnitUs);
      if (cost < best - 1e-9) {
        best = cost;
        bn = kCand[i];
      }
    }
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
    case 192: return launch_qgemm_bn<192>(tm_xq, tm_bcat, tm_ucat, a, st);
    case 256: return launch_qgemm_bn<256>(tm_xq, tm_bcat, tm_ucat, a, st);
    default: return cudaErrorInvalidValue;
  }
}

UgemmPlan plan_ugemm(int T, int K, int R_tot) {
  UgemmPlan p;
  if (R_tot <= 256) p.nu = R_tot;
  else if (R_tot % 256 == 0) p.nu = 256;
  else if (R_tot % 192 == 0) p.nu = 192;
  else if (R_tot % 128 == 0) p.nu = 128;
  else p.nu = 64;
  p.ntiles = static_cast<int>(ceil_div(R_tot, p.nu));
  const int mtiles = static_cast<int>(ceil_div(T, 128));
  const int nk = static_cast<int>(ceil_div(K, kAdapterAtom));
  // about two waves of CTAs, each with at least 4 K chunks
  int splits = static_cast<int>(ceil_div(2 * 148, int64_t(mtiles) * p.ntiles));
  splits = std::max(1, std::min(splits, std::max(1, nk / 4)));
  p.kchunks_per_split = static_cast<int>(ceil_div(nk, splits));
  p.splits = static_cast<int>(ceil_div(nk, p.kchunks_per_split));
  return p;
}

cudaError_t launch_ugemm(const CUtensorMap& tm_x, const CUtensorMap& tm_acat, const UgemmPlan& plan, int T, int K,
                         int R_tot, float* partial, unsigned* zero_ctr, int* err, cudaStream_t st) {
  switch (plan.nu) {
#define QE_NU(n) \
  case n: return launch_ugemm_t<n>(tm_x, tm_acat, plan, T, K, R_tot, partial, zero_ctr, err, st);
    QE_NU(16) QE_NU(32) QE_NU(48) QE_NU(80) QE_NU(144) QE_NU(208) QE_NU(64) QE_NU(128) QE_NU(192) QE_NU(256)
#undef QE_NU
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qe
