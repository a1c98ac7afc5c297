// Weight-only product (W4A16 / W3A16) of the QE linear layer on the tensor cores.
//
// Y[p][o] = sum_j sw[o,j] * sum_{k in group j} bf16(x_p[k]*s_inv[k]) * q[o,k]  +  su[p] * (U_cat . B_cat^T)
//
// The weight codes q are small integers, exact in bf16, and the activations are the bf16 values
// the layer is defined on, so every product is exact in the fp32 accumulator. One TMEM buffer per
// quantization group holds that group's sum; the epilogue scales it by sw and adds it in fp32,
// the same factorisation as the int8 path. The tile is M = 128 output channels (TMEM lanes) by
// N = BN token positions in bucket order (BN <= 64: decode-sized batches; larger batches take
// more token tiles). Warp roles (512 threads):
//   warp 0      bulk copies of the packed weight blocks into their own ring (8 KB slots), so
//               the HBM stream runs ahead of the unpacking
//   warp 3      TMA loads of the activation tile (two 64-wide K atoms) into the operand slot,
//               and of the adapter operands after the last block of a unit
//   warps 8-15  unpack 3- or 4-bit codes into bf16 in the 128B-swizzled A layout of the slot
//   warps 1-2   one thread each issues tcgen05.mma kind::f16 (bf16) for alternate blocks, 8 K
//               steps per 128-deep block; the first step of a group starts a fresh accumulator
//   warps 4-7   epilogue: per group acc += sw * tmem; at the end of a unit + su * adapter,
//               then a scatter of the rows to token order through shared memory
// Unpacking writes bf16(128 + u) with a byte permute (u = the code's offset-binary value) and
// subtracts 128 + offset in bf16x2, which is exact for these integers.
#include <cuda_bf16.h>

#include <algorithm>
#include <utility>

#include "qe_internal.h"
#include "qe_ptx.cuh"

namespace qe {
namespace {

template <int BN>
struct WCfg {
  static constexpr int kAtomA = 16384;   // 128 rows x 64 bf16
  static constexpr int kA = 2 * kAtomA;  // one 128-deep K block
  static constexpr int kAtomB = BN * 128;
  static constexpr int kB = 2 * kAtomB;
  static constexpr int kSlot = kA + kB;
  // Operand slots: each holds a 32 KB bf16 weight tile, so they bound the blocks in flight
  // between unpacking and the MMA; narrow tiles leave room for one more.
  static constexpr int kNA = (BN <= 32) ? 4 : (BN <= 64 ? 3 : 2);
  static constexpr int kNW = 6;                 // packed weight ring
  static constexpr int kWP = 8192;
  static constexpr int kNB = (BN <= 64) ? 8 : 4;  // TMEM accumulator buffers (fp32, BN columns each)
  static_assert(kNB % 2 == 0, "each MMA issuer owns half of the buffers");
  // Roles (512 threads): warp 0 weight blocks, warps 1-2 MMA issuers, warp 3 activation tiles,
  // then the epilogue warps, then the unpack warps. 128-token tiles take a second team of 4
  // epilogue warps from the unpack warps: each team keeps half of the tile's columns in
  // registers, and 4 unpack warps convert a row each.
  static constexpr int kThreads = 512;
  static constexpr int kEpiWarps = (BN <= 64) ? 4 : 8;
  static constexpr int kUnpackW0 = 4 + kEpiWarps;
  static constexpr int kUnpackWarps = 16 - kUnpackW0;
  static constexpr int kEC = BN * 4 / kEpiWarps;  // columns per epilogue thread
  static constexpr int kTmemCols = (kNB * BN <= 128) ? 128 : (kNB * BN <= 256 ? 256 : 512);
  static constexpr int kOut = (BN <= 32) ? 8192 : 16384;  // output staging
  static constexpr int kChunk = (BN >= 16) ? 16 : BN;
  static constexpr size_t kSmem =
      1024 + size_t(kNA) * kSlot + size_t(kNW) * kWP + kOut + 1024 + size_t(BN) * 8;
  static_assert(kSmem <= 232448, "shared memory");
};

struct WUnit {
  int nt, p0, split, kb_begin, nkb, n_ad, g_begin, n_groups;
};

__device__ __forceinline__ WUnit make_wunit(const QgemmArgs& a, int BN, int u) {
  WUnit w;
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
  w.g_begin = w.kb_begin * gpb;
  w.n_groups = max(0, min(a.K / a.group, kb_end * gpb) - w.g_begin);
  return w;
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t x, uint32_t y) {
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&y);
  __nv_bfloat162 r = __hsub2(a, b);
  return *reinterpret_cast<uint32_t*>(&r);
}

// Four 4-bit two's-complement codes held in the byte lanes of v (one nibble per byte, at `shift`)
// -> four bf16 values, little-endian, in two words.
__device__ __forceinline__ uint2 w4_to_bf16(uint32_t v, int shift) {
  const uint32_t u = ((v >> shift) & 0x0F0F0F0Fu) ^ 0x08080808u;  // q + 8 in [1, 15]
  const uint32_t bias = 0x43084308u;                               // bf16(136) twice
  const uint32_t lo = __byte_perm(u, 0x00004300u, 0x5150);          // bf16(128 + u0), bf16(128 + u1)
  const uint32_t hi = __byte_perm(u, 0x00004300u, 0x5352);          // bf16(128 + u2), bf16(128 + u3)
  return make_uint2(bf16x2_sub(lo, bias), bf16x2_sub(hi, bias));
}

// Two 3-bit offset-binary codes u = q + 4: low two bits at bits [lo_shift, +2) and [16 + lo_shift, +2)
// of lw, bit 2 at bits hi_shift and 16 + hi_shift of hw -> bf16 pair (q_even, q_odd). Two
// three-input logic ops build bf16(128 + u) in both halves; one bf16x2 subtraction leaves q.
__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));  // (a & b) | c
  return d;
}
__device__ __forceinline__ uint32_t w3_pair_to_bf16(uint32_t lw, uint32_t hw, int lo_shift, int hi_shift) {
  const uint32_t l = lop3_and_or(lw >> lo_shift, 0x00030003u, 0x43004300u);  // bf16(128 + low bits)
  const uint32_t hs = (hi_shift >= 2) ? (hw >> (hi_shift - 2)) : (hw << (2 - hi_shift));
  const uint32_t bf = lop3_and_or(hs, 0x00040004u, l);                        // + 4 * bit 2
  return bf16x2_sub(bf, 0x43044304u);                                         // - bf16(132)
}

template <int BITS, int BN>
__global__ void __launch_bounds__(512, 1)
    k_wgemm(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_bcat,
            const __grid_constant__ CUtensorMap tm_ucat, const QgemmArgs a) {
  using C = WCfg<BN>;
  constexpr int NA = C::kNA, NW = C::kNW, NB = C::kNB;
  constexpr int kBlock = (BITS == 4) ? kW4BlockBytes : kW3BlockBytes;
  int* const a_err = a.err;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* slots = smem;                           // [NA][A | B]
  uint8_t* wring = slots + NA * C::kSlot;          // [NW][8 KB]
  uint8_t* out_stage = wring + NW * C::kWP;        // [16 KB]
  uint64_t* bars = reinterpret_cast<uint64_t*>(out_stage + C::kOut);
  uint64_t* wfull = bars;             // [NW] packed block landed
  uint64_t* wempty = wfull + NW;      // [NW] unpack warps read it (one arrival per unpack warp)
  uint64_t* afull = wempty + NW;      // [NA] A unpacked (one arrival per unpack warp)
  uint64_t* aempty = afull + NA;      // [NA] MMAs done with the slot
  uint64_t* accf = aempty + NA;       // [NB] group sum ready
  uint64_t* acce = accf + NB;         // [NB] group sum read (every epilogue warp)
  uint64_t* done = acce + NB;
  uint64_t* adone = done + 1;         // adapter block: its issuer waited for all of its slots
  uint64_t* aack = adone + 1;         // adapter block: the other issuer saw adone
  uint64_t* bfull = aack + 1;         // [NA] the slot's TMA tiles landed (1 + bytes)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bfull + NA);
  float* su_s = reinterpret_cast<float*>(bars + 64);
  int32_t* perm_s = reinterpret_cast<int32_t*>(su_s + BN);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NT = static_cast<int>(ceil_div(a.N, kTileN));
  const int PT = static_cast<int>(ceil_div(a.T, BN));
  const int n_units = NT * PT * a.splits;
  const int gpb = kTileK / a.group;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NW; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], C::kUnpackWarps);
    }
    for (int s = 0; s < NA; ++s) {
      mbar_init(&afull[s], C::kUnpackWarps);
      mbar_init(&bfull[s], 1);
      mbar_init(&aempty[s], 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], C::kEpiWarps);
    }
    mbar_init(done, 2);
    mbar_init(adone, 1);
    mbar_init(aack, 1);
    mbar_arrive(aack);  // phase 0: nothing to acknowledge before the first adapter block
    mbar_fence_init();
    prefetch_tmap(&tm_act);
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
  grid_dep_wait();
  grid_dep_launch();

  if (warp == 0) {
    // ------------------------------------------------------------ packed weight blocks
    if (lane == 0) {
      int jw = 0;
      for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        const WUnit w = make_wunit(a, BN, u);
        bool ok = true;
        for (int i = 0; i < w.nkb; ++i, ++jw) {
          const int s = jw % NW;
          if (!mbar_wait(&wempty[s], ((jw / NW) & 1) ^ 1, a_err, DEVERR_WAIT_PRODUCER)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&wfull[s], kBlock);
          bulk_load(wring + s * C::kWP, a.w_packed + (static_cast<size_t>(w.nt) * a.KB + w.kb_begin + i) * kBlock,
                    kBlock, &wfull[s]);
        }
        if (!ok) break;
      }
      drain_ring(wfull, NW, jw);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ activation / adapter tiles
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const WUnit w = make_wunit(a, BN, u);
        for (int i = 0; i < w.nkb + w.n_ad; ++i, ++it) {
          const int s = it % NA;
          if (!mbar_wait(&aempty[s], ((it / NA) & 1) ^ 1, a_err, DEVERR_WAIT_PRODUCER)) {
            ok = false;
            break;
          }
          uint8_t* sa_ = slots + s * C::kSlot;
          uint8_t* sb_ = sa_ + C::kA;
          if (i < w.nkb) {
            const int k0 = (w.kb_begin + i) * kTileK;
            mbar_arrive_expect_tx(&bfull[s], C::kB);
            tma_load_2d(sb_, &tm_act, k0, w.p0, &bfull[s]);
            tma_load_2d(sb_ + C::kAtomB, &tm_act, k0 + 64, w.p0, &bfull[s]);
          } else {
            const int at = i - w.nkb;
            mbar_arrive_expect_tx(&bfull[s], C::kAtomA + C::kAtomB);
            tma_load_2d(sa_, &tm_bcat, at * kAdapterAtom, w.nt * kTileN, &bfull[s]);
            tma_load_2d(sb_, &tm_ucat, at * kAdapterAtom, w.p0, &bfull[s]);
          }
        }
      }
      drain_ring(bfull, NA, it);
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    // Two threads issue alternate blocks: one thread's issue rate, not the tensor pipe, limits
    // these narrow (BN <= 64) MMAs. A unit's adapter atoms accumulate into one TMEM buffer, so
    // one issuer takes all of them. Parity waits stay within one phase of their barrier as in
    // the int8 kernel: issuer q owns TMEM buffers q, q+2, ..., and an issuer that skipped an
    // adapter block waits on adone (the owner waited for every slot of the block) before its
    // next slot; the owner of the next block first waits on aack.
    const int qi = warp - 1;
    if (lane == 0) {
      const uint32_t id_bf = idesc_bf16(128, BN);
      const uint32_t id_ad = idesc_f16(128, BN);
      const uint64_t desc_a0 = smem_desc_sw128(smem_u32(slots));
      constexpr int kOwn = NB / 2;  // TMEM buffers per issuer
      int it = 0;
      uint32_t own = 0, ablk = 0;  // groups this issuer took (mod 8), adapter blocks seen (mod 2)
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const WUnit w = make_wunit(a, BN, u);
        const int ad_owner = (it + w.nkb) & 1;
        for (int i = 0; i < w.nkb + w.n_ad && ok; ++i, ++it) {
          const int s = it % NA;
          const uint64_t da = desc_a0 + static_cast<uint64_t>((s * C::kSlot) >> 4);
          const uint64_t db = da + (C::kA >> 4);
          if (i < w.nkb) {
            const int kb = w.kb_begin + i;
            const int ng = max(0, min(gpb, w.g_begin + w.n_groups - kb * gpb));
            if ((it & 1) != qi) continue;
            if (!mbar_wait(&afull[s], (it / NA) & 1, a_err, DEVERR_WAIT_MMA) ||
                !mbar_wait(&bfull[s], (it / NA) & 1, a_err, DEVERR_WAIT_MMA)) {
              ok = false;
              break;
            }
            // 8 K steps of 16 per block (4 per 64-wide atom): one group (g = 128) or two (g = 64)
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
              const int k_first = (gpb == 1) ? 0 : 4 * gi, k_count = (gpb == 1) ? 8 : 4;
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                if (kk >= k_count) break;
                const int ks = k_first + kk;  // K step of 16 inside the block
                const uint64_t off = static_cast<uint64_t>((ks >> 2) * (C::kAtomA >> 4) + (ks & 3) * 2);
                const uint64_t offb = static_cast<uint64_t>((ks >> 2) * (C::kAtomB >> 4) + (ks & 3) * 2);
                mma_f16(d, da + off, db + offb, id_bf, kk > 0 ? 1u : 0u);
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
            if (!mbar_wait(&afull[s], (it / NA) & 1, a_err, DEVERR_WAIT_MMA) ||
                !mbar_wait(&bfull[s], (it / NA) & 1, a_err, DEVERR_WAIT_MMA)) {
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
          tc_commit(&aempty[s]);
          if (i >= w.nkb && i - w.nkb == w.n_ad - 1) {
            // this issuer owned the adapter block and has waited for all of its slots
            if (!mbar_wait(aack, ablk, a_err, DEVERR_WAIT_MMA)) {
              ok = false;
              break;
            }
            mbar_arrive(adone);
            ablk ^= 1u;
          }
        }
      }
      tc_commit(done);
      mbar_wait(done, 0, a_err, DEVERR_WAIT_TEARDOWN);
    }
  } else if (warp >= C::kUnpackW0) {
    // ------------------------------------------------------------ unpack
    // 8 warps: thread t takes row r = t/2 of the block and the 64-wide K atom t%2 of it.
    // 4 warps: thread t takes row t, both atoms.
    constexpr int kAtomsPerThread = C::kUnpackWarps == 8 ? 1 : 2;
    const int ut = threadIdx.x - 32 * C::kUnpackW0;
    const int r = kAtomsPerThread == 1 ? ut >> 1 : ut;
    int it = 0, jw = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const WUnit w = make_wunit(a, BN, u);
      for (int i = 0; i < w.nkb + w.n_ad; ++i, ++it) {
        const int s = it % NA;
        if (i < w.nkb) {
          const int ws = jw % NW;
          if (!mbar_wait(&wfull[ws], (jw / NW) & 1, a_err, DEVERR_WAIT_UNPACK) ||
              !mbar_wait(&aempty[s], ((it / NA) & 1) ^ 1, a_err, DEVERR_WAIT_UNPACK)) {
            ok = false;
            break;
          }
          const uint8_t* src = wring + ws * C::kWP;
#pragma unroll
          for (int ai = 0; ai < kAtomsPerThread; ++ai) {
          const int atom = kAtomsPerThread == 1 ? (ut & 1) : ai;
          uint8_t* dst = slots + s * C::kSlot + atom * C::kAtomA + r * 128;
          if constexpr (BITS == 4) {
            // row r: 64 bytes, four 16-byte pieces; this atom is pieces 2*atom and 2*atom+1
            const uint4 p0 = *reinterpret_cast<const uint4*>(src + r * 64 + atom * 32);
            const uint4 p1 = *reinterpret_cast<const uint4*>(src + r * 64 + atom * 32 + 16);
            const uint32_t pw[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
            for (int pc = 0; pc < 2; ++pc) {
              // piece pc: low nibbles of words 0..3 -> atom K 32pc + 0..15 (chunks 4pc, 4pc+1),
              // high nibbles -> 32pc + 16..31 (chunks 4pc+2, 4pc+3)
#pragma unroll
              for (int half = 0; half < 2; ++half) {
#pragma unroll
                for (int wp2 = 0; wp2 < 2; ++wp2) {
                  const uint2 e0 = w4_to_bf16(pw[4 * pc + 2 * wp2], 4 * half);
                  const uint2 e1 = w4_to_bf16(pw[4 * pc + 2 * wp2 + 1], 4 * half);
                  const int ch = 4 * pc + 2 * half + wp2;
                  *reinterpret_cast<uint4*>(dst + ((ch ^ (r & 7)) << 4)) = make_uint4(e0.x, e0.y, e1.x, e1.y);
                }
              }
            }
          } else {
            // row r: 48 bytes; low two bits in words m = 4*atom + 0..3, bit 2 in words h = 2*atom + 0..1
            const uint4 lq = *reinterpret_cast<const uint4*>(src + r * 48 + atom * 16);
            const uint2 hq = *reinterpret_cast<const uint2*>(src + r * 48 + 32 + atom * 8);
            const uint32_t lw[4] = {lq.x, lq.y, lq.z, lq.w};
            const uint32_t hw[2] = {hq.x, hq.y};
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
              // chunk ch = atom K 8ch..8ch+7: low word ch/2 (pairs p = 4*(ch&1) + 0..3), high word ch/4
              // (pairs p' = 4*(ch&3) + 0..3)
              uint32_t e[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int p = 4 * (ch & 1) + j, ph = 4 * (ch & 3) + j;
                e[j] = w3_pair_to_bf16(lw[ch >> 1], hw[ch >> 2], 2 * p, ph);
              }
              *reinterpret_cast<uint4*>(dst + ((ch ^ (r & 7)) << 4)) = make_uint4(e[0], e[1], e[2], e[3]);
            }
          }
          }
          // free the packed block only now: its values have been used, so every load from it has
          // completed before the next bulk copy can land in the slot
          __syncwarp();
          if (lane == 0) mbar_arrive(&wempty[ws]);
          fence_proxy_async_smem();
          ++jw;
        } else {
          if (!mbar_wait(&aempty[s], ((it / NA) & 1) ^ 1, a_err, DEVERR_WAIT_UNPACK)) {
            ok = false;
            break;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[s]);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue (warps 4..4+kEpiWarps)
    // Control flow depends only on the unit schedule; after a wait runs out, `ok` turns every
    // later wait and TMEM access off (the named barrier below is still reached by all).
    constexpr int EC = C::kEC, NE = 32 * C::kEpiWarps;
    const int q = warp & 3;
    const int team = C::kEpiWarps == 8 ? (warp - 4) >> 2 : 0;
    const int ch0 = team * EC;          // this team's first column
    const int et = threadIdx.x - 128;   // 0..NE-1
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    // group -> TMEM buffer as the issuers assign it (issuer of the block's parity, its buffers in turn)
    constexpr int kOwn = NB / 2;
    uint32_t bstate = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
      const WUnit w = make_wunit(a, BN, u);
      const int o0 = w.nt * kTileN;
      const int o = o0 + 32 * q + lane;
      const bool o_ok = o < a.N;
      asm volatile("bar.sync 2, %0;" ::"n"(NE) : "memory");
      for (int c = et; c < BN; c += NE) {
        const int p = w.p0 + c;
        su_s[c] = (p < a.T && a.su_sorted) ? a.su_sorted[p] : 0.0f;
        perm_s[c] = (p < a.T) ? a.perm[p] : -1;
      }
      asm volatile("bar.sync 2, %0;" ::"n"(NE) : "memory");
      float acc[EC];
#pragma unroll
      for (int c = 0; c < EC; ++c) acc[c] = 0.0f;
      const size_t sw0 = static_cast<size_t>(w.g_begin) * a.N + o;  // scale of (o, first group)
      float sw_next = (o_ok && w.n_groups > 0) ? load_scale(a.w_scale, sw0, a.sw_f16) : 0.0f;
      for (int g = 0; g < w.n_groups; ++g) {
        uint32_t use;
        const int b = epi_next_buffer<kOwn>(bstate, static_cast<int>(bstate & 1u), use);
        // bit 0 follows the stage parity: flip it after the last group of each K block
        if (a.group == kTileK || (g & 1) || g + 1 == w.n_groups) bstate ^= 1u;
        const float sw = sw_next;
        if (o_ok && g + 1 < w.n_groups) sw_next = load_scale(a.w_scale, sw0 + static_cast<size_t>(g + 1) * a.N, a.sw_f16);
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&accf[b], use & 1, a_err, DEVERR_WAIT_EPILOGUE));
        if (!ok) continue;
        tc_fence_after();
        const uint32_t base = tmem + lane_base + b * BN + ch0;
#pragma unroll
        for (int c = 0; c < EC; c += C::kChunk) {
          uint32_t v[C::kChunk];
          if constexpr (C::kChunk == 16) tmem_ld16(base + c, v);
          else tmem_ld8(base + c, v);
          tmem_wait_ld();
          reg_fence(v);
#pragma unroll
          for (int i = 0; i < C::kChunk; ++i) acc[c + i] = fmaf(sw, __uint_as_float(v[i]), acc[c + i]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[b]);
      }
      if (w.n_ad > 0) {
        uint32_t use;
        const int b = epi_next_buffer<kOwn>(bstate, static_cast<int>(bstate & 1u), use);
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&accf[b], use & 1, a_err, DEVERR_WAIT_EPILOGUE));
        if (ok) {
          tc_fence_after();
          const uint32_t base = tmem + lane_base + b * BN + ch0;
#pragma unroll
          for (int c = 0; c < EC; c += C::kChunk) {
            uint32_t v[C::kChunk];
            if constexpr (C::kChunk == 16) tmem_ld16(base + c, v);
            else tmem_ld8(base + c, v);
            tmem_wait_ld();
            reg_fence(v);
#pragma unroll
            for (int i = 0; i < C::kChunk; ++i)
              acc[c + i] = fmaf(su_s[ch0 + c + i], __uint_as_float(v[i]), acc[c + i]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acce[b]);
        }
      }
      // store: each pass moves PC columns through the staging buffer, then whole row segments
      // (128 channels) go to Y[perm[p]] (or row p of this split's partial buffer)
      const bool to_partial = a.splits > 1;
      const bool bf = !to_partial && a.y_bf16;
      const int row_bytes = bf ? 256 : 512;
      const int PC = C::kOut / row_bytes < BN ? C::kOut / row_bytes : BN;
      const int elem = bf ? 2 : 4;
      const bool vec_ok = ((static_cast<size_t>(a.N) * elem) % 16) == 0;
      for (int pass = 0; pass < BN / PC; ++pass) {
#pragma unroll
        for (int cc = 0; cc < EC; ++cc) {
          const int c = ch0 + cc;
          if (c < pass * PC || c >= (pass + 1) * PC) continue;
          const int cl = c - pass * PC;
          if (bf) {
            __nv_bfloat16 h = __float2bfloat16_rn(acc[cc]);
            *reinterpret_cast<__nv_bfloat16*>(out_stage + cl * row_bytes + (32 * q + lane) * 2) = h;
          } else {
            *reinterpret_cast<float*>(out_stage + cl * row_bytes + (32 * q + lane) * 4) = acc[cc];
          }
        }
        asm volatile("bar.sync 2, %0;" ::"n"(NE) : "memory");
        if (ok) {
          const int chunks_per_row = row_bytes / 16, elems = 16 / elem;
          for (int ch = et; ch < PC * chunks_per_row; ch += NE) {
            const int cl = ch / chunks_per_row, part = ch % chunks_per_row;
            const int col = pass * PC + cl;
            const int p = w.p0 + col;
            const int row = to_partial ? (p < a.T ? p : -1) : perm_s[col];
            if (row < 0) continue;
            const int of = o0 + part * elems;
            if (of >= a.N) continue;
            uint8_t* dst = to_partial
                               ? reinterpret_cast<uint8_t*>(a.partial + (static_cast<size_t>(w.split) * a.T + row) * a.N)
                               : static_cast<uint8_t*>(a.Y) + static_cast<size_t>(row) * a.N * elem;
            const uint8_t* srcp = out_stage + cl * row_bytes + part * 16;
            if (vec_ok && of + elems <= a.N) {
              *reinterpret_cast<uint4*>(dst + static_cast<size_t>(of) * elem) = *reinterpret_cast<const uint4*>(srcp);
            } else {
              for (int e = 0; e < elems && of + e < a.N; ++e) {
                if (elem == 2)
                  *reinterpret_cast<uint16_t*>(dst + static_cast<size_t>(of + e) * 2) =
                      *reinterpret_cast<const uint16_t*>(srcp + e * 2);
                else
                  *reinterpret_cast<float*>(dst + static_cast<size_t>(of + e) * 4) =
                      *reinterpret_cast<const float*>(srcp + e * 4);
              }
            }
          }
        }
        asm volatile("bar.sync 2, %0;" ::"n"(NE) : "memory");
      }
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

template <int BITS, int BN>
cudaError_t launch_wgemm_t(const CUtensorMap& tm_act, const CUtensorMap& tm_bcat, const CUtensorMap& tm_ucat,
                           const QgemmArgs& a, cudaStream_t st) {
  using C = WCfg<BN>;
  cudaError_t e = cudaFuncSetAttribute(k_wgemm<BITS, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  static int n_sm = 0;
  if (n_sm == 0) {
    int dev = 0;
    cudaError_t ed = cudaGetDevice(&dev);
    if (ed == cudaSuccess) ed = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (ed != cudaSuccess) return ed;
  }
  const int64_t units = ceil_div(a.N, kTileN) * ceil_div(a.T, BN) * a.splits;
  const unsigned grid = static_cast<unsigned>(units < n_sm ? units : n_sm);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_wgemm<BITS, BN>, tm_act, tm_bcat, tm_ucat, a);
}


}  // namespace

int pick_wgemm_bn(int T, int N, int K, int* splits_out, int* kbps_out) {
  // a weight block is unpacked once per token tile: wide tiles once there are enough tiles
  const int64_t nt = ceil_div(N, kTileN);
  const int bn = (T <= 16) ? 16 : (T <= 32 ? 32 : ((T <= 64 || nt * ceil_div(T, 128) < 148) ? 64 : 128));
  const int ntiles = static_cast<int>(ceil_div(N, kTileN));
  const int KB = static_cast<int>(ceil_div(K, kTileK));
  const int64_t tiles = int64_t(ntiles) * ceil_div(T, bn);
  // split K until every SM has a unit (decode layers are a single token tile)
  int splits = 1;
  if (tiles < 148 && KB >= 8) splits = static_cast<int>(std::min<int64_t>(KB / 4, ceil_div(2 * 148, tiles)));
  if (splits < 1) splits = 1;
  const int kbps = static_cast<int>(ceil_div(KB, splits));
  *splits_out = static_cast<int>(ceil_div(KB, kbps));
  *kbps_out = kbps;
  return bn;
}

cudaError_t launch_wgemm(int bits, int BN, const CUtensorMap& tm_act, const CUtensorMap& tm_bcat,
                         const CUtensorMap& tm_ucat, const QgemmArgs& a, cudaStream_t st) {
  if (bits == 4) {
    if (BN == 16) return launch_wgemm_t<4, 16>(tm_act, tm_bcat, tm_ucat, a, st);
    if (BN == 32) return launch_wgemm_t<4, 32>(tm_act, tm_bcat, tm_ucat, a, st);
    if (BN == 64) return launch_wgemm_t<4, 64>(tm_act, tm_bcat, tm_ucat, a, st);
    if (BN == 128) return launch_wgemm_t<4, 128>(tm_act, tm_bcat, tm_ucat, a, st);
  } else if (bits == 3) {
    if (BN == 16) return launch_wgemm_t<3, 16>(tm_act, tm_bcat, tm_ucat, a, st);
    if (BN == 32) return launch_wgemm_t<3, 32>(tm_act, tm_bcat, tm_ucat, a, st);
    if (BN == 64) return launch_wgemm_t<3, 64>(tm_act, tm_bcat, tm_ucat, a, st);
    if (BN == 128) return launch_wgemm_t<3, 128>(tm_act, tm_bcat, tm_ucat, a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace qe
