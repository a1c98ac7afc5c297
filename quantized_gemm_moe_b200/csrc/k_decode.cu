// Product of a decode-sized batch (T <= 16 tokens) of the QE linear layer on the tensor cores.
//
// At T <= 16 the layer streams the packed weights once and does little arithmetic per byte, so
// HBM bandwidth bounds it (the 72B decode layers move ~120 MB of codes for 16 tokens). The
// prefill kernels tile by output block and split K only when tiles are scarce; here the whole
// (output tile, K block) sequence is split evenly over the SMs instead ("stream-K"): CTA c takes
// blocks [c*NB/G, (c+1)*NB/G) of the tile-major order, so every SM streams the same number of
// bytes whatever the shape. A CTA's range crosses at most a few tile boundaries; each piece of a
// tile (a segment) leaves an fp32 partial, and the CTA that finishes a tile's last segment adds the
// tile's partials in segment order (deterministic), applies the token scale and the adapter term,
// and writes Y.
//
// Per 128 x 128 weight block:
//   warp 0      bulk copies of the packed block and of its group-scale slabs, and TMA of the
//               activation tile (16 tokens x 128 channels), into a 14-16 deep ring: up to 128 KB
//               of weights in flight per SM. The epilogue frees a slot once it has read the scales.
//   warps 4-11  unpack the block straight into tensor memory with tcgen05.st: the MMA takes its
//               A operand (the weights, M = 128 output rows = TMEM lanes, K along the columns)
//               from TMEM, so the unpacked weights never pass through shared memory (whose
//               bandwidth the unpack would otherwise exceed at the HBM rate). Two teams of four
//               warps (one per TMEM lane quarter) take alternate blocks, a full row per thread.
//   warps 1-2   one thread each issues the MMAs of alternate blocks: kind::i8 (codes x16 against
//               int8 activation codes, 4 K steps) or kind::f16 (bf16 weights against bf16
//               activations, 8 K steps). Every quantization group gets a fresh 16-column
//               accumulator (the first K step does not accumulate), issuer q owning slots
//               q, q+2, ...
//   warp 3      the adapter term U_cat . B_catT of every tile whose first block this CTA streams,
//               on CUDA cores (fp16 inputs, fp32 sums), written to the workspace off the epilogue's path
//   warps 12-15 epilogue, one output row per thread: per group acc += sw * group sum (the int8
//               sums converted exactly, the scale read from the ring slot); the segment partials
//               and the per-tile fix-up.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "qe_internal.h"
#include "qe_ptx.cuh"

namespace qe {
namespace {

constexpr int kDN = 16;          // token columns: the whole batch, padded (MMA N)
constexpr int kDThreads = 512;   // 16 warps
constexpr int kDTmemCols = 512;

template <bool I8, int BITS>
struct DCfg {
  static constexpr int kWBlock = (BITS == 4) ? kW4BlockBytes : kW3BlockBytes;
  static constexpr int kXAtom = kDN * 128;                // 16 rows x 128 bytes (one swizzle atom pair)
  static constexpr int kXTile = I8 ? kXAtom : 2 * kXAtom;  // 128 input channels: int8 codes or bf16
  static constexpr int kACols = I8 ? 32 : 64;             // TMEM columns of one unpacked block
  static constexpr int kKSteps = I8 ? 4 : 8;              // MMA K steps per block (32 int8 / 16 bf16)
  // unpacked A blocks in TMEM: the loop unpack -> MMA -> slot free spans this many blocks
  static constexpr int kASlots = I8 ? 8 : 6;
  static constexpr int kAccSlots = (kDTmemCols - kASlots * kACols) / kDN;  // 16 (int8) / 8 (bf16)
  static constexpr int kOwn = kAccSlots / 2;              // accumulator slots per issuer
  static constexpr int kUcatBytes = kDN * 512 * 2;        // U_cat staging, R_pad <= 512
  static constexpr int kSBlock = 2 * 128 * 4;             // group scale slabs of a block (2 groups x 128 rows)
  // Three rings, all even so that each unpack team / issuer keeps its own slots:
  //  packed blocks: freed by the unpack team as soon as it has used them, so the HBM stream only
  //    waits on one hand-off (load -> unpack);
  //  activation tiles: freed by the MMA commit;  scale slabs: freed by the epilogue.
  // The last two recycle later in the pipeline, so they are deeper (and small).
  static constexpr int kWStages = (I8 || BITS == 3) ? 16 : 12;
  static constexpr int kXStages = I8 ? 24 : 16;
  static constexpr int kSStages = I8 ? 24 : 16;
  static constexpr size_t kSmem = 1024 + size_t(kXStages) * kXTile + size_t(kWStages) * kWBlock +
                                  size_t(kSStages) * kSBlock + kUcatBytes + 1024;
  static_assert(kWStages % 2 == 0 && kXStages % 2 == 0 && kSStages % 2 == 0, "team / issuer owned ring slots");
  static_assert(kAccSlots % 2 == 0, "each issuer owns half of the accumulator slots");
  static_assert(kASlots % 2 == 0, "each unpack team and issuer keeps its own A slots");
  static_assert(kSmem <= 232448, "shared memory");
};

struct DecArgs {
  const uint8_t* w_packed;
  const float* w_scale;     // [G][N] fp32, or fp16 when sw_f16
  int sw_f16, sw_elem;      // scale bytes: 4 or 2
  int sw_vec;               // N * sw_elem is a multiple of 16: slabs travel with the blocks
  const float* sa_sorted;   // [T]
  const float* su_sorted;   // [T] or nullptr (no adapters)
  const int32_t* perm;      // [T]
  const uint16_t* ucat;     // fp16 [T][R_pad], bucket order
  const uint16_t* bcat;     // fp16 [N][R_pad]
  int R_pad;
  int T, N, K, group, KB, NT, G_total;
  int64_t NB;               // NT * KB
  int maxseg;
  void* Y;
  int y_bf16;
  float* part;              // [NT][maxseg][128][16]
  float* ad;                // [NT][128][16]
  unsigned* cnt;            // [NT], zero at launch
  int32_t* dbg_acc;         // [T][N][G] token order, or nullptr
  int* err;
};

// CTA c of G owns blocks [range_begin(c), range_begin(c+1)) of the NB blocks in tile-major order;
// block f belongs to CTA cta_of(f).
__host__ __device__ __forceinline__ int64_t range_begin(int c, int64_t NB, int G) {
  return static_cast<int64_t>(c) * NB / G;
}
__host__ __device__ __forceinline__ int cta_of(int64_t f, int64_t NB, int G) {
  return static_cast<int>(((f + 1) * G - 1) / NB);
}

// (output tile, K block) of consecutive blocks, advanced without divisions (a 64-bit division per
// block costs hundreds of cycles on a role's critical path).
struct BlockPos {
  int nt, kb;
  __device__ __forceinline__ void next(int KB) {
    if (++kb == KB) {
      kb = 0;
      ++nt;
    }
  }
};

__device__ __forceinline__ void mma_i8_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t x, uint32_t y) {
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&y);
  __nv_bfloat162 r = __hsub2(a, b);
  return *reinterpret_cast<uint32_t*>(&r);
}
// Four 4-bit two's-complement codes (one nibble per byte, at `shift`) -> bf16 pairs (q0,q1), (q2,q3):
// bf16(128 + q + 8) built by a byte permute, then bf16(136) subtracted (exact for these integers).
__device__ __forceinline__ uint2 w4_to_bf16(uint32_t v, int shift) {
  const uint32_t u = ((v >> shift) & 0x0F0F0F0Fu) ^ 0x08080808u;
  const uint32_t lo = __byte_perm(u, 0x00004300u, 0x5150);
  const uint32_t hi = __byte_perm(u, 0x00004300u, 0x5352);
  return make_uint2(bf16x2_sub(lo, 0x43084308u), bf16x2_sub(hi, 0x43084308u));
}
__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));  // (a & b) | c
  return d;
}
// Two 3-bit offset-binary codes u = q + 4 (low two bits at lo_shift and 16 + lo_shift of lw, bit 2
// at hi_shift and 16 + hi_shift of hw) -> the bf16 pair (q_even, q_odd).
__device__ __forceinline__ uint32_t w3_pair_to_bf16(uint32_t lw, uint32_t hw, int lo_shift, int hi_shift) {
  const uint32_t l = lop3_and_or(lw >> lo_shift, 0x00030003u, 0x43004300u);
  const uint32_t hs = (hi_shift >= 2) ? (hw >> (hi_shift - 2)) : (hw << (2 - hi_shift));
  return bf16x2_sub(lop3_and_or(hs, 0x00040004u, l), 0x43044304u);
}

__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// One thread's half row (64 input channels) of block rows r, unpacked into TMEM columns
// [col, col + kACols/2) of its lane: the A operand layout (row = lane, K along the columns, four
// int8 or two bf16 per 32-bit column, lowest channel in the low bits).
template <bool I8, int BITS>
__device__ __forceinline__ void unpack_half_row(const uint8_t* blk, int r, int half, uint32_t taddr) {
  if constexpr (BITS == 4) {
    // row r: four 16-byte pieces; piece i holds channels 32i..32i+15 in the low nibbles of its words
    // (word w: channels 32i+4w..+3) and 32i+16..32i+31 in the high nibbles
    const uint4 p0 = *reinterpret_cast<const uint4*>(blk + r * 64 + half * 32);
    const uint4 p1 = *reinterpret_cast<const uint4*>(blk + r * 64 + half * 32 + 16);
    const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    if constexpr (I8) {
      // the code goes to the high nibble of its byte: the byte is the int8 16*q (the x16 is folded
      // into the group scale)
      uint32_t v[16];
#pragma unroll
      for (int pc = 0; pc < 2; ++pc)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[8 * pc + j] = (w[4 * pc + j] << 4) & 0xF0F0F0F0u;
          v[8 * pc + 4 + j] = w[4 * pc + j] & 0xF0F0F0F0u;
        }
      tmem_st_x16(taddr, v);
    } else {
#pragma unroll
      for (int pc = 0; pc < 2; ++pc) {
        uint32_t v[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint2 lo = w4_to_bf16(w[4 * pc + j], 0), hi = w4_to_bf16(w[4 * pc + j], 4);
          v[2 * j] = lo.x;
          v[2 * j + 1] = lo.y;
          v[8 + 2 * j] = hi.x;
          v[8 + 2 * j + 1] = hi.y;
        }
        tmem_st_x16(taddr + 16 * pc, v);
      }
    }
  } else {
    // row r: 48 bytes; column c (channels 2c, 2c+1) of this half: low word 4*half + (c%32)/8 at
    // pair c%8, high word 2*half + (c%32)/16 at pair c%16
    const uint4 lq = *reinterpret_cast<const uint4*>(blk + r * 48 + half * 16);
    const uint2 hq = *reinterpret_cast<const uint2*>(blk + r * 48 + 32 + half * 8);
    const uint32_t lw[4] = {lq.x, lq.y, lq.z, lq.w};
    const uint32_t hw[2] = {hq.x, hq.y};
#pragma unroll
    for (int pc = 0; pc < 2; ++pc) {
      uint32_t v[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int c = 16 * pc + j;
        v[j] = w3_pair_to_bf16(lw[c >> 3], hw[c >> 4], 2 * (c & 7), c & 15);
      }
      tmem_st_x16(taddr + 16 * pc, v);
    }
  }
}

template <bool I8, int BITS>
__global__ void __launch_bounds__(kDThreads, 1)
    k_qdec(const __grid_constant__ CUtensorMap tm_x, const DecArgs a) {
  using C = DCfg<I8, BITS>;
  constexpr int NW = C::kWStages, NX = C::kXStages, NSS = C::kSStages, NA = C::kASlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xring = smem;                              // [NX][kXTile], 1024-aligned (128B swizzle)
  uint8_t* wring = xring + NX * C::kXTile;            // [NW][kWBlock]
  uint8_t* sring = wring + NW * C::kWBlock;           // [NSS][2 groups][128 rows] group scales
  __half* ucat_s = reinterpret_cast<__half*>(sring + NSS * C::kSBlock);  // [16][R_pad]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(ucat_s) + C::kUcatBytes);
  uint64_t* wfull = bars;                  // [NW] packed block landed (1 + bytes)
  uint64_t* wempty = wfull + NW;           // [NW] the unpack team has used it (4 warps)
  uint64_t* xfull = wempty + NW;           // [NX] activation tile landed (1 + bytes)
  uint64_t* xempty = xfull + NX;           // [NX] the block's MMAs are done
  uint64_t* sfull = xempty + NX;           // [NSS] scale slabs landed (1 + bytes)
  uint64_t* sempty = sfull + NSS;          // [NSS] the epilogue read them (4 warps)
  uint64_t* afull = sempty + NSS;          // [NA] A unpacked into TMEM (the 4 warps of a team)
  uint64_t* aempty = afull + NA;           // [NA] the MMAs of the block are done (A slot free)
  uint64_t* accf = aempty + NA;            // [kAccSlots] group sum ready
  uint64_t* acce = accf + C::kAccSlots;    // [kAccSlots] group sum read (4 epilogue warps)
  uint64_t* done = acce + C::kAccSlots;    // teardown
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* flag_s = reinterpret_cast<int*>(tmem_slot + 1);
  volatile int* ad_done = reinterpret_cast<volatile int*>(tmem_slot + 2);  // adapter tiles written so far

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const int64_t b0 = range_begin(c, a.NB, G), b1 = range_begin(c + 1, a.NB, G);
  const int nblk = static_cast<int>(b1 - b0);
  const int gpb = kTileK / a.group;
  const BlockPos pos0{static_cast<int>(b0 / a.KB), static_cast<int>(b0 % a.KB)};
  int* const a_err = a.err;
  // tiles whose first block lies in this CTA's range: their adapter terms are computed here
  const int nt_ad0 = static_cast<int>((b0 + a.KB - 1) / a.KB), nt_ad1 = static_cast<int>((b1 - 1) / a.KB);
  const bool any_ad = a.su_sorted != nullptr && nt_ad0 <= nt_ad1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NW; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 4);
    }
    for (int s = 0; s < NX; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1);
    }
    for (int s = 0; s < NSS; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 4);
    }
    *ad_done = 0;
    for (int s = 0; s < NA; ++s) {
      mbar_init(&afull[s], 4);
      mbar_init(&aempty[s], 1);
    }
    for (int b = 0; b < C::kAccSlots; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 4);
    }
    mbar_init(done, 2);
    mbar_fence_init();
    prefetch_tmap(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kDTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t colA = 0, colAcc = NA * C::kACols;
  grid_dep_wait();
  grid_dep_launch();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // per block: the packed block, its activation tile and its scale slabs, each into its own ring
    if (lane == 0) {
      int i = 0;
      BlockPos bp = pos0;
      bool ok = true;
      for (; i < nblk; ++i, bp.next(a.KB)) {
        const int kb = bp.kb;
        const int sw = i % NW, sx = i % NX, ss = i % NSS;
        if (!mbar_wait(&wempty[sw], ((i / NW) & 1) ^ 1, a_err, DEVERR_WAIT_PRODUCER)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&wfull[sw], C::kWBlock);
        bulk_load(wring + sw * C::kWBlock, a.w_packed + (b0 + i) * C::kWBlock, C::kWBlock, &wfull[sw]);
        if (!mbar_wait(&xempty[sx], ((i / NX) & 1) ^ 1, a_err, DEVERR_WAIT_PRODUCER)) {
          ok = false;
          ++i;
          break;
        }
        mbar_arrive_expect_tx(&xfull[sx], C::kXTile);
        tma_load_2d(xring + sx * C::kXTile, &tm_x, kb * kTileK, 0, &xfull[sx]);
        if constexpr (!I8) tma_load_2d(xring + sx * C::kXTile + C::kXAtom, &tm_x, kb * kTileK + 64, 0, &xfull[sx]);
        if (!mbar_wait(&sempty[ss], ((i / NSS) & 1) ^ 1, a_err, DEVERR_WAIT_PRODUCER)) {
          ok = false;
          ++i;
          break;
        }
        // the 128-row scale slab of each of the block's groups (contiguous: group-major [G][N]);
        // with a row pitch that is not a multiple of 16 bytes the epilogue reads its scales itself
        const int ng = min(gpb, a.G_total - kb * gpb);
        const int o0 = bp.nt * kTileN;
        const uint32_t scopy = a.sw_vec ? static_cast<uint32_t>(min(128, a.N - o0) * a.sw_elem) : 0u;
        mbar_arrive_expect_tx(&sfull[ss], ng * scopy);
        for (int gi = 0; gi < (scopy ? ng : 0); ++gi)
          bulk_load(sring + ss * C::kSBlock + gi * 512,
                    reinterpret_cast<const uint8_t*>(a.w_scale) +
                        (static_cast<size_t>(kb * gpb + gi) * a.N + o0) * a.sw_elem,
                    scopy, &sfull[ss]);
      }
      (void)ok;
      drain_ring(wfull, NW, i);
      drain_ring(xfull, NX, i);
      drain_ring(sfull, NSS, i);
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers (alternate blocks)
    const int qi = warp - 1;
    if (lane == 0) {
      const uint32_t idesc = I8 ? idesc_i8(128, kDN) : idesc_bf16(128, kDN);
      const uint64_t xdesc0 = smem_desc_sw128(smem_u32(xring));
      int own = 0;
      bool ok = true;
      BlockPos bp = pos0;
      if (qi) bp.next(a.KB);
      for (int i = qi; i < nblk && ok; i += 2, bp.next(a.KB), bp.next(a.KB)) {
        const int sx = i % NX, as = i % NA;
        const int kb = bp.kb;
        const int ng = min(gpb, a.G_total - kb * gpb);
        if (!mbar_wait(&afull[as], (i / NA) & 1, a_err, DEVERR_WAIT_MMA) ||
            !mbar_wait(&xfull[sx], (i / NX) & 1, a_err, DEVERR_WAIT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t xdesc = xdesc0 + static_cast<uint64_t>((sx * C::kXTile) >> 4);
        const uint32_t a_col = tmem + colA + as * C::kACols;
        for (int gi = 0; gi < ng; ++gi) {
          const int slot = qi + 2 * (own % C::kOwn);
          const uint32_t use = static_cast<uint32_t>(own / C::kOwn);
          ++own;
          if (!mbar_wait(&acce[slot], (use & 1u) ^ 1u, a_err, DEVERR_WAIT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + colAcc + slot * kDN;
          const int k0 = (gpb == 1) ? 0 : gi * (C::kKSteps / 2);
          const int nk = (gpb == 1) ? C::kKSteps : C::kKSteps / 2;
          for (int kk = 0; kk < nk; ++kk) {
            const int ks = k0 + kk;
            if constexpr (I8) {
              // K step of 32 int8: 8 TMEM columns of A, 32 bytes along the tile's swizzled rows
              mma_i8_ta(d, a_col + ks * 8, xdesc + static_cast<uint64_t>(2 * ks), idesc, kk > 0 ? 1u : 0u);
            } else {
              // K step of 16 bf16: 8 TMEM columns of A; the tile is two 64-channel atoms
              const uint64_t offb = static_cast<uint64_t>((ks >> 2) * (C::kXAtom >> 4) + (ks & 3) * 2);
              mma_f16_ta(d, a_col + ks * 8, xdesc + offb, idesc, kk > 0 ? 1u : 0u);
            }
          }
          tc_commit(&accf[slot]);
        }
        tc_commit(&aempty[as]);
        tc_commit(&xempty[sx]);
      }
      tc_commit(done);
      mbar_wait(done, 0, a_err, DEVERR_WAIT_TEARDOWN);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ adapter terms (CUDA cores)
    // ad[nt][r][p] = sum_j B_catT[o][j] * U_cat[p][j] (fp16 inputs, fp32 sums) for every tile whose
    // first block this CTA streams; lane l takes rows l, l+32, l+64, l+96. Off the epilogue's path:
    // the segment holding a tile's first block waits for that tile's term (the count ad_done)
    // only when it finishes.
    if (any_ad) {
      const int rp = a.R_pad, T = a.T;
      for (int e = lane; e < kDN * rp / 8; e += 32) {
        const int p = e / (rp / 8), c8 = e % (rp / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (p < T) v = __ldg(reinterpret_cast<const uint4*>(a.ucat + static_cast<size_t>(p) * rp) + c8);
        *reinterpret_cast<uint4*>(ucat_s + static_cast<size_t>(p) * rp + c8 * 8) = v;
      }
      __syncwarp();
      for (int nt = nt_ad0; nt <= nt_ad1; ++nt) {
        for (int rr = 0; rr < 4; ++rr) {
          const int r = lane + 32 * rr;
          const int o = nt * kTileN + r;
          float adr[kDN];
#pragma unroll
          for (int p = 0; p < kDN; ++p) adr[p] = 0.0f;
          if (o < a.N) {
            const uint4* brow = reinterpret_cast<const uint4*>(a.bcat + static_cast<size_t>(o) * rp);
            for (int c0 = 0; c0 < rp / 8; c0 += 8) {
              uint4 bv[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) bv[k] = (c0 + k < rp / 8) ? __ldg(brow + c0 + k) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                if (c0 + k >= rp / 8) break;
                const __half2* bh = reinterpret_cast<const __half2*>(&bv[k]);
                float2 bf[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) bf[q] = __half22float2(bh[q]);
#pragma unroll
                for (int p = 0; p < kDN; ++p) {
                  if (p >= T) break;
                  const uint4 uv = *reinterpret_cast<const uint4*>(ucat_s + static_cast<size_t>(p) * rp + (c0 + k) * 8);
                  const __half2* uh = reinterpret_cast<const __half2*>(&uv);
                  float sacc = adr[p];
#pragma unroll
                  for (int q = 0; q < 4; ++q) {
                    const float2 uf = __half22float2(uh[q]);
                    sacc = fmaf(bf[q].x, uf.x, sacc);
                    sacc = fmaf(bf[q].y, uf.y, sacc);
                  }
                  adr[p] = sacc;
                }
              }
            }
          }
          float4* dst = reinterpret_cast<float4*>(a.ad + (static_cast<size_t>(nt) * kTileN + r) * kDN);
#pragma unroll
          for (int k = 0; k < kDN / 4; ++k) dst[k] = make_float4(adr[4 * k], adr[4 * k + 1], adr[4 * k + 2], adr[4 * k + 3]);
        }
        // this tile's term is in memory: the epilogue can finish the tile's first segment
        __threadfence();
        __syncwarp();
        if (lane == 0) *ad_done = nt - nt_ad0 + 1;
      }
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ unpack into TMEM
    // Two teams of four warps (one per TMEM lane quarter) take alternate blocks, so two blocks are
    // in flight; each thread unpacks one full row of the block.
    const int q4 = warp & 3, team = (warp - 4) >> 2;
    const int r = 32 * q4 + lane;  // block row = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * q4) << 16;
    for (int i = team; i < nblk; i += 2) {
      const int sw = i % NW, as = i % NA;
      if (!mbar_wait(&wfull[sw], (i / NW) & 1, a_err, DEVERR_WAIT_UNPACK) ||
          !mbar_wait(&aempty[as], ((i / NA) & 1) ^ 1, a_err, DEVERR_WAIT_UNPACK))
        break;
      tc_fence_after();
      const uint32_t ta = tmem + lane_base + colA + as * C::kACols;
      unpack_half_row<I8, BITS>(wring + sw * C::kWBlock, r, 0, ta);
      unpack_half_row<I8, BITS>(wring + sw * C::kWBlock, r, 1, ta + C::kACols / 2);
      // the packed block's values have been used (the stores below hold them): free its slot now,
      // so the next load can land while this block goes through the MMA
      __syncwarp();
      if (lane == 0) mbar_arrive(&wempty[sw]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[as]);
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ epilogue, one output row per thread
    // Control flow follows the block schedule only; after a wait ran out, `ok` turns off every
    // later wait and TMEM access, and the named barriers are still reached by all four warps.
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;
    const int et = threadIdx.x - 384;  // 0..127
    const uint32_t lane_base = static_cast<uint32_t>(32 * q4) << 16;
    const int T = a.T;
    // the group scales of block i: the 128-row slab(s) the producer copied into ring slot i % NS
    // (or, when a row of scales is not a multiple of 16 bytes, this thread's own scale from memory)
    auto scale_at = [&](int s, int gi, int nt, int j) -> float {
      if (a.sw_vec) {
        const uint8_t* slab = sring + s * C::kSBlock + gi * 512;
        if (a.sw_f16) return __half2float(*reinterpret_cast<const __half*>(slab + r * 2));
        return *reinterpret_cast<const float*>(slab + r * 4);
      }
      const int o = nt * kTileN + r;
      return (o < a.N) ? load_scale(a.w_scale, static_cast<size_t>(j) * a.N + o, a.sw_f16) : 0.0f;
    };

    bool ok = true;
    int cnt0 = 0, cnt1 = 0;  // groups drained from issuer 0 / 1
    float acc[kDN];
#pragma unroll
    for (int p = 0; p < kDN; ++p) acc[p] = 0.0f;
    int cur_nt = -1;
    bool cur_ad = false;     // this segment holds its tile's first block

    // End of a segment of tile nt: a tile held by this CTA alone is written at once; otherwise the
    // partial goes to its slot and the last CTA to finish the tile adds the partials in segment order.
    auto finish_segment = [&](int nt, bool has_first) {
      const int64_t f0 = static_cast<int64_t>(nt) * a.KB;
      const int c_first = cta_of(f0, a.NB, G);
      const int nseg = cta_of(f0 + a.KB - 1, a.NB, G) - c_first + 1;
      const int seg = c - c_first;
      const int o = nt * kTileN + r;
      const size_t tile_row = (static_cast<size_t>(nt) * kTileN + r) * kDN;
      // the adapter term of this tile was computed by warp 3 of this CTA
      if (has_first && a.su_sorted && ok) {
        // warp 3 writes the terms in tile order; this is tile nt - nt_ad0 of that list
        const int need = nt - nt_ad0 + 1;
        bool got = *ad_done >= need;
        if (!got) {
          const uint64_t t0 = globaltimer_ns();
          while (!(got = (*ad_done >= need)) && globaltimer_ns() - t0 < kWaitLimitNs) __nanosleep(256);
        }
        if (!got) record_error(a_err, DEVERR_WAIT_EPILOGUE);
        __threadfence_block();
        ok = __all_sync(0xffffffffu, got);
      }
      bool last = true;
      if (nseg > 1) {
        float4* dst = reinterpret_cast<float4*>(a.part + (static_cast<size_t>(nt) * a.maxseg + seg) * kTileN * kDN +
                                                static_cast<size_t>(r) * kDN);
#pragma unroll
        for (int k = 0; k < kDN / 4; ++k) dst[k] = make_float4(acc[4 * k], acc[4 * k + 1], acc[4 * k + 2], acc[4 * k + 3]);
        __threadfence();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (et == 0) {
          const unsigned old = atomicAdd(a.cnt + nt, 1u);
          *flag_s = (old == static_cast<unsigned>(nseg - 1)) ? 1 : 0;
          __threadfence();
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        last = *flag_s != 0;
        if (last) {
#pragma unroll
          for (int p = 0; p < kDN; ++p) acc[p] = 0.0f;
          for (int sgi = 0; sgi < nseg; ++sgi) {
            const float4* src = reinterpret_cast<const float4*>(
                a.part + (static_cast<size_t>(nt) * a.maxseg + sgi) * kTileN * kDN + static_cast<size_t>(r) * kDN);
#pragma unroll
            for (int k = 0; k < kDN / 4; ++k) {
              const float4 v = __ldcg(src + k);
              acc[4 * k] += v.x;
              acc[4 * k + 1] += v.y;
              acc[4 * k + 2] += v.z;
              acc[4 * k + 3] += v.w;
            }
          }
        }
      }
      if (last) {
        float adr[kDN];
#pragma unroll
        for (int p = 0; p < kDN; ++p) adr[p] = 0.0f;
        if (a.su_sorted) {
          const float4* ad = reinterpret_cast<const float4*>(a.ad + tile_row);
#pragma unroll
          for (int k = 0; k < kDN / 4; ++k) {
            const float4 v = __ldcg(ad + k);
            adr[4 * k] = v.x;
            adr[4 * k + 1] = v.y;
            adr[4 * k + 2] = v.z;
            adr[4 * k + 3] = v.w;
          }
        }
        if (o < a.N) {
#pragma unroll
          for (int p = 0; p < kDN; ++p) {
            if (p >= T) break;
            // int8 codes carry the token scale; weight-only layers computed with the bf16 activation itself
            float y = I8 ? acc[p] * __ldg(a.sa_sorted + p) : acc[p];
            if (a.su_sorted) y = fmaf(__ldg(a.su_sorted + p), adr[p], y);
            const size_t at = static_cast<size_t>(__ldg(a.perm + p)) * a.N + o;
            if (a.y_bf16) {
              static_cast<__nv_bfloat16*>(a.Y)[at] = __float2bfloat16_rn(y);
            } else {
              static_cast<float*>(a.Y)[at] = y;
            }
          }
        }
        if (nseg > 1 && et == 0) a.cnt[nt] = 0u;  // leave the counter at zero for the next launch
      }
    };

    BlockPos bp = pos0;
    for (int i = 0; i < nblk; ++i, bp.next(a.KB)) {
      const int nt = bp.nt, kb = bp.kb;
      if (nt != cur_nt) {
        if (cur_nt >= 0) finish_segment(cur_nt, cur_ad);
        cur_nt = nt;
        cur_ad = kb == 0;
#pragma unroll
        for (int p = 0; p < kDN; ++p) acc[p] = 0.0f;
      }
      // this block's scale slabs (the phase cannot move on before this epilogue frees the slot,
      // so the parity wait is exact)
      const int ss = i % NSS;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&sfull[ss], (i / NSS) & 1, a_err, DEVERR_WAIT_EPILOGUE));
      const float s0 = scale_at(ss, 0, nt, kb * gpb);
      const float s1 = (gpb == 2) ? scale_at(ss, 1, nt, kb * gpb + 1) : 0.0f;
      const int q = i & 1;
      const int ng = min(gpb, a.G_total - kb * gpb);
      for (int gi = 0; gi < ng; ++gi) {
        const int n_q = q ? cnt1 : cnt0;
        const int slot = q + 2 * (n_q % C::kOwn);
        const uint32_t use = static_cast<uint32_t>(n_q / C::kOwn);
        if (q) ++cnt1;
        else ++cnt0;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&accf[slot], use & 1u, a_err, DEVERR_WAIT_EPILOGUE));
        if (!ok) continue;
        tc_fence_after();
        uint32_t v[kDN];
        tmem_ld16(tmem + lane_base + colAcc + slot * kDN, v);
        tmem_wait_ld();
        reg_fence(v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[slot]);
        const float sw = gi ? s1 : s0;
        if constexpr (I8) {
          const float swq = sw * 0.0625f;  // codes entered the MMA as 16*q
#pragma unroll
          for (int p = 0; p < kDN; ++p) acc[p] = fmaf(static_cast<float>(static_cast<int32_t>(v[p])), swq, acc[p]);
          if (a.dbg_acc) {
            const int o = nt * kTileN + r;
            if (o < a.N) {
#pragma unroll
              for (int p = 0; p < kDN; ++p) {
                if (p >= T) break;
                a.dbg_acc[(static_cast<size_t>(__ldg(a.perm + p)) * a.N + o) * a.G_total + kb * gpb + gi] =
                    static_cast<int32_t>(v[p]) / 16;
              }
            }
          }
        } else {
#pragma unroll
          for (int p = 0; p < kDN; ++p) acc[p] = fmaf(__uint_as_float(v[p]), sw, acc[p]);
        }
      }
      // the block's scales have been read: the slot can take a later block's
      __syncwarp();
      if (lane == 0) mbar_arrive(&sempty[ss]);
    }
    if (cur_nt >= 0) finish_segment(cur_nt, cur_ad);
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kDTmemCols);
  }
}

template <bool I8, int BITS>
cudaError_t launch_qdec_t(const CUtensorMap& tm_x, const DecArgs& a, int grid, cudaStream_t st) {
  using C = DCfg<I8, BITS>;
  cudaError_t e = cudaFuncSetAttribute(k_qdec<I8, BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kDThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_qdec<I8, BITS>, tm_x, a);
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
                                                   cudaSuccess)
      n = 0;
  }
  return n;
}

}  // namespace

DecodePlan plan_decode(int N, int K, int n_sm) {
  DecodePlan p;
  p.NT = static_cast<int>(ceil_div(N, kTileN));
  p.KB = static_cast<int>(ceil_div(K, kTileK));
  p.NB = int64_t(p.NT) * p.KB;
  p.grid = static_cast<int>(std::min<int64_t>(p.NB, n_sm > 0 ? n_sm : 148));
  // a tile of KB consecutive blocks meets at most (KB - 1) / Lmin + 2 of the ranges (Lmin >= 1 blocks each)
  const int64_t lmin = p.NB / p.grid;
  p.maxseg = static_cast<int>((p.KB - 1) / lmin + 2);
  p.part_bytes = size_t(p.NT) * p.maxseg * kTileN * kDN * 4;
  p.ad_bytes = size_t(p.NT) * kTileN * kDN * 4;
  p.cnt_words = p.NT;
  return p;
}

int decode_grid_sms() { return sm_count(); }

cudaError_t launch_qdec(int w_bits, bool int8, const CUtensorMap& tm_x, const DecodePlan& plan,
                        const QgemmArgs& q, const uint16_t* ucat, const uint16_t* bcat, int R_pad, float* part,
                        float* ad, unsigned* cnt, cudaStream_t st) {
  DecArgs a{};
  a.w_packed = q.w_packed;
  a.w_scale = q.w_scale;
  a.sw_f16 = q.sw_f16;
  a.sw_elem = q.sw_f16 ? 2 : 4;
  a.sw_vec = ((static_cast<int64_t>(q.N) * a.sw_elem) % 16) == 0 ? 1 : 0;
  a.sa_sorted = q.sa_sorted;
  a.su_sorted = q.su_sorted;
  a.perm = q.perm;
  a.ucat = ucat;
  a.bcat = bcat;
  a.R_pad = R_pad;
  a.T = q.T;
  a.N = q.N;
  a.K = q.K;
  a.group = q.group;
  a.KB = plan.KB;
  a.NT = plan.NT;
  a.G_total = q.K / q.group;
  a.NB = plan.NB;
  a.maxseg = plan.maxseg;
  a.Y = q.Y;
  a.y_bf16 = q.y_bf16;
  a.part = part;
  a.ad = ad;
  a.cnt = cnt;
  a.dbg_acc = q.dbg_acc;
  a.err = q.err;
  if (q.T > kDN || q.T < 1 || R_pad > 512) return cudaErrorInvalidValue;
  if (int8) {
    if (w_bits != 4) return cudaErrorInvalidValue;
    return launch_qdec_t<true, 4>(tm_x, a, plan.grid, st);
  }
  if (w_bits == 4) return launch_qdec_t<false, 4>(tm_x, a, plan.grid, st);
  if (w_bits == 3) return launch_qdec_t<false, 3>(tm_x, a, plan.grid, st);
  return cudaErrorInvalidValue;
}

}  // namespace qe
