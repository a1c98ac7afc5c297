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
// At 16 tokens a 128 x 128 block carries little work for any role, so the fixed cost of each
// hand-off decides the speed: an MMA or a commit keeps its issuing thread ~140 cycles whatever N
// is (several issuing threads overlap), and every dependent barrier step of a role costs a few
// hundred cycles. The roles are laid out to keep those steps few per byte:
//   warp 0      bulk copy of each packed block into a 16-20 deep ring (120-160 KB in flight per
//               SM), freed by the unpack team as soon as it has read the block. No earlier kernel
//               writes the weights, so the stream starts before the previous grid has finished.
//   warps 4-11  unpack the block straight into tensor memory with tcgen05.st: the MMA takes its
//               A operand (the weights, M = 128 output rows = TMEM lanes, K along the columns)
//               from TMEM, so the unpacked weights never pass through shared memory. Two teams of
//               four warps (one per TMEM lane quarter) take alternate blocks, a row per thread.
//   warps 1-3   one thread each issues the MMAs of every third block: kind::i8 (codes x16 against
//               int8 activation codes, 4 K steps) or kind::f16 (bf16 weights against bf16
//               activations, 8 K steps), one commit per block (frees the block's A slot). Each
//               also loads the activation tiles (16 tokens x 128 channels, TMA) of its own blocks
//               six blocks ahead, into a 12-slot ring.
//               Every quantization group gets a fresh 16-column accumulator; eight (bf16: four)
//               consecutive groups share one batch buffer (two buffers), committed once per batch.
//   warps 12-15 epilogue, one output row per thread, a batch of groups at a time: the group
//               sums (int8 sums converted exactly) times the group scales (each thread copies its
//               own with cp.async, three batches ahead), the segment partials and the per-tile
//               fix-up, which adds su times
//               the adapter term U_cat . B_catT of the tile. The adapter terms of the tiles whose
//               first block this CTA streams are computed by these threads while the pipeline fills.
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
constexpr int kMaxRpad = kDecodeMaxRpad;  // adapter rank (padded) the decode product takes
constexpr int kIssuers = 3;      // MMA issuing threads (warps 1-3): an MMA keeps its thread ~140 cycles

template <bool I8, int BITS>
struct DCfg {
  static constexpr int kWBlock = (BITS == 4) ? kW4BlockBytes : kW3BlockBytes;
  static constexpr int kXAtom = kDN * 128;                // 16 rows x 128 bytes (one swizzle atom pair)
  static constexpr int kXTile = I8 ? kXAtom : 2 * kXAtom;  // 128 input channels: int8 codes or bf16
  static constexpr int kACols = I8 ? 32 : 64;             // TMEM columns of one unpacked block
  static constexpr int kKSteps = I8 ? 4 : 8;              // MMA K steps per block (32 int8 / 16 bf16)
  // unpacked blocks in TMEM: unpack -> MMA -> slot free spans this many blocks. A multiple of 6,
  // so that each of the two unpack teams and each of the three issuers keeps its own slots.
  static constexpr int kASlots = 6;
  static constexpr int kBatch = I8 ? 8 : 4;               // groups per epilogue batch (16 columns each)
  static constexpr int kBufs = 2;                         // batch buffers
  static constexpr int kXSlots = 2 * kASlots;             // activation tiles: block i's tile in slot i % 12
  static constexpr int kWStages = (I8 || BITS == 3) ? 20 : 16;  // packed-block ring
  static constexpr int kScaleBatches = 4;                 // scale ring: batches in flight + the one in use
  static constexpr size_t kSmem = 1024 + size_t(kXSlots) * kXTile + size_t(kWStages) * kWBlock +
                                  size_t(kDN) * kMaxRpad * 4 + size_t(kScaleBatches) * kBatch * kTileN * 4 + 1024;
  static_assert(kASlots * kACols + kBufs * kBatch * kDN <= kDTmemCols, "tensor memory");
  static_assert(kWStages % 2 == 0 && kASlots % 6 == 0, "each unpack team / issuer keeps its own slots");
  static_assert(kSmem <= 232448, "shared memory");
};

struct DecArgs {
  const uint8_t* w_packed;
  const float* w_scale;     // [G][N] fp32, or fp16 when sw_f16
  int sw_f16;
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

// Walks the quantization groups of consecutive blocks: block position, group within the block and
// groups of the block (the last K block of a ragged K holds fewer).
struct GroupPos {
  BlockPos bp;
  int gi, ng;
  __device__ __forceinline__ void init(BlockPos p, int gpb, int G_total) {
    bp = p;
    gi = 0;
    ng = min(gpb, G_total - p.kb * gpb);
  }
  __device__ __forceinline__ void next(int KB, int gpb, int G_total) {
    if (++gi == ng) {
      gi = 0;
      bp.next(KB);
      ng = min(gpb, G_total - bp.kb * gpb);
    }
  }
};

// ad[nt][r][p] = sum_j B_catT[nt*128 + r][j] * U_cat[p][j] for p < T (zero for p >= T and rows past
// d_out): the adapter term of row r of tile nt, fp16 inputs (U_cat staged as fp32 in u_s) and fp32
// sums. The row is read eight 16-byte pieces at a time, all in flight together.
__device__ __forceinline__ void adapter_row(const DecArgs& a, const float* u_s, int nt, int r) {
  const int o = nt * kTileN + r;
  float acc[kDN];
#pragma unroll
  for (int p = 0; p < kDN; ++p) acc[p] = 0.0f;
  const uint4* brow = reinterpret_cast<const uint4*>(a.bcat + static_cast<size_t>(o) * a.R_pad);
  const int n8 = (o < a.N) ? a.R_pad / 8 : 0;
  for (int c0 = 0; c0 < n8; c0 += 8) {
    uint4 bv[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) bv[k] = (c0 + k < n8) ? __ldg(brow + c0 + k) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const __half2* bh = reinterpret_cast<const __half2*>(&bv[k]);
      float bf[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __half22float2(bh[q]);
        bf[2 * q] = f.x;
        bf[2 * q + 1] = f.y;
      }
      const int j0 = min(c0 + k, n8 - 1) * 8;  // pieces past the row are zero: any in-range U column
#pragma unroll
      for (int p = 0; p < kDN; ++p) {
        const float4 u0 = *reinterpret_cast<const float4*>(u_s + p * a.R_pad + j0);
        const float4 u1 = *reinterpret_cast<const float4*>(u_s + p * a.R_pad + j0 + 4);
        float t = acc[p];
        t = fmaf(bf[0], u0.x, t);
        t = fmaf(bf[1], u0.y, t);
        t = fmaf(bf[2], u0.z, t);
        t = fmaf(bf[3], u0.w, t);
        t = fmaf(bf[4], u1.x, t);
        t = fmaf(bf[5], u1.y, t);
        t = fmaf(bf[6], u1.z, t);
        t = fmaf(bf[7], u1.w, t);
        acc[p] = t;
      }
    }
  }
  float4* dst = reinterpret_cast<float4*>(a.ad + (static_cast<size_t>(nt) * kTileN + r) * kDN);
#pragma unroll
  for (int k = 0; k < kDN / 4; ++k) dst[k] = make_float4(acc[4 * k], acc[4 * k + 1], acc[4 * k + 2], acc[4 * k + 3]);
}

template <bool I8, int BITS>
__global__ void __launch_bounds__(kDThreads, 1)
    k_qdec(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ DecArgs a) {
  using C = DCfg<I8, BITS>;
  constexpr int NW = C::kWStages, NA = C::kASlots, NX = C::kXSlots, NBUF = C::kBufs, NBATCH = C::kBatch;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xring = smem;                              // [NX][kXTile], 1024-aligned (128B swizzle)
  uint8_t* wring = xring + NX * C::kXTile;            // [NW][kWBlock]
  float* u_s = reinterpret_cast<float*>(wring + NW * C::kWBlock);  // U_cat as fp32 [16][R_pad]
  uint32_t* sc_s = reinterpret_cast<uint32_t*>(u_s + kDN * kMaxRpad);  // [4][NBATCH][128] scale words
  uint64_t* bars = reinterpret_cast<uint64_t*>(sc_s + C::kScaleBatches * NBATCH * kTileN);
  uint64_t* wfull = bars;          // [NW] packed block landed (1 + bytes)
  uint64_t* wempty = wfull + NW;   // [NW] the unpack team has read it (4 warps)
  uint64_t* xfull = wempty + NW;   // [NX] activation tile landed (1 + bytes)
  uint64_t* afull = xfull + NX;    // [NA] block unpacked into TMEM (the 4 warps of a team)
  uint64_t* mdone = afull + NA;    // [NA] the block's MMAs are done: its A slot is free
  uint64_t* accf = mdone + NA;     // [NBUF] batch of group sums ready (one commit per issuer)
  uint64_t* acce = accf + NBUF;    // [NBUF] batch read (4 epilogue warps)
  uint64_t* done = acce + NBUF;    // teardown
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* flag_s = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const int64_t b0 = range_begin(c, a.NB, G), b1 = range_begin(c + 1, a.NB, G);
  const int nblk = static_cast<int>(b1 - b0);
  const int gpb = kTileK / a.group;
  const BlockPos pos0{static_cast<int>(b0 / a.KB), static_cast<int>(b0 % a.KB)};
  // groups of this CTA's blocks (with a ragged K the last K block of each tile holds fewer) and
  // the epilogue batches they form
  const bool ragged = a.G_total < a.KB * gpb;
  const int ngroups = nblk * gpb - (ragged ? static_cast<int>(b1 / a.KB - b0 / a.KB) : 0);
  const int nbatch = (ngroups + NBATCH - 1) / NBATCH;
  int* const a_err = a.err;

  {
    // one barrier per thread (the arrays are contiguous: wfull, wempty, xfull, afull, mdone, accf,
    // acce, done)
    constexpr int kBars = 2 * NW + NX + 2 * NA + 2 * NBUF + 1;
    static_assert(kBars <= kDThreads, "one thread per barrier");
    const int t = threadIdx.x;
    if (t < kBars) {
      int count = 1;  // wfull, xfull, mdone: one arrival (+ bytes / commit)
      if ((t >= NW && t < 2 * NW) || (t >= 2 * NW + NX && t < 2 * NW + NX + NA)) count = 4;  // wempty, afull
      if (t >= 2 * NW + NX + 2 * NA) {
        const int u = t - (2 * NW + NX + 2 * NA);  // accf[NBUF], acce[NBUF], done
        count = (u < NBUF) ? kIssuers : (u < 2 * NBUF) ? 4 : kIssuers;
      }
      mbar_init(&bars[t], static_cast<uint32_t>(count));
      mbar_fence_init();
    }
    if (t == kBars) prefetch_tmap(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kDTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t colA = 0, colAcc = NA * C::kACols;  // A slots, then the batch buffers
  grid_dep_launch();

  if (warp == 0) {
    // ------------------------------------------------------------ packed blocks
    // No earlier kernel writes the packed weights, so this warp streams them without waiting for
    // the previous grid.
    if (lane == 0) {
      int i = 0;
      for (; i < nblk; ++i) {
        const int s = i % NW;
        if (!mbar_wait(&wempty[s], ((i / NW) & 1) ^ 1, a_err, DEVERR_WAIT_PRODUCER)) break;
        mbar_arrive_expect_tx(&wfull[s], C::kWBlock);
        bulk_load(wring + s * C::kWBlock, a.w_packed + (b0 + i) * C::kWBlock, C::kWBlock, &wfull[s]);
      }
      drain_ring(wfull, NW, i);
    }
  } else if (warp >= 1 && warp <= kIssuers) {
    // ------------------------------------------------------------ MMA issuers (every third block)
    const int qi = warp - 1;
    grid_dep_wait();  // the activation tiles are the previous grid's output
    if (lane == 0) {
      // Each issuer loads the activation tiles of its own blocks, NA blocks ahead. Block j's tile
      // goes to slot j % NX, which last held block j - NX's; it is requested once this issuer has
      // seen afull of block j - NA, whose A slot the unpack team refilled only after the MMAs of
      // block j - 2 NA = j - NX were done. Blocks j and j - NA have the same issuer.
      int ix = qi;             // next own block whose tile is requested
      BlockPos xb = pos0;      // position of block ix
      for (int t = 0; t < qi; ++t) xb.next(a.KB);
      auto request_tile = [&]() {
        const int s = ix % NX;
        mbar_arrive_expect_tx(&xfull[s], C::kXTile);
        tma_load_2d(xring + s * C::kXTile, &tm_x, xb.kb * kTileK, 0, &xfull[s]);
        if constexpr (!I8) tma_load_2d(xring + s * C::kXTile + C::kXAtom, &tm_x, xb.kb * kTileK + 64, 0, &xfull[s]);
        ix += kIssuers;
        for (int t = 0; t < kIssuers; ++t) xb.next(a.KB);
      };
      while (ix < nblk && ix < NA) request_tile();  // the first NA blocks' tiles: slots never used
      const uint32_t idesc = I8 ? idesc_i8(128, kDN) : idesc_bf16(128, kDN);
      const uint64_t xdesc0 = smem_desc_sw128(smem_u32(xring));
      bool ok = true;
      int acquired = 0;   // batches whose buffer this issuer has waited for (in order)
      int committed = 0;  // batches this issuer has committed (in order)
      // the buffer of batch b is free once the epilogue has drained batch b - NBUF
      auto acquire = [&](int b) {
        while (ok && acquired <= b) {
          ok = mbar_wait(&acce[acquired % NBUF], ((acquired / NBUF) & 1) ^ 1, a_err, DEVERR_WAIT_MMA);
          if (ok) {
            tc_fence_after();
            ++acquired;
          }
        }
      };
      // this issuer has issued all its groups of the batches before b: one commit each (a batch
      // is committed only after its buffer was acquired, so an arrival never lands in the
      // barrier's previous phase)
      auto commit_before = [&](int b) {
        while (ok && committed < b) {
          acquire(committed);
          if (!ok) break;
          tc_commit(&accf[committed % NBUF]);
          ++committed;
        }
      };
      BlockPos bp = pos0;
      int gidx = 0;  // first group of block i in this CTA's group sequence
      for (int i = 0; i < nblk && ok; ++i, bp.next(a.KB)) {
        const int ng = min(gpb, a.G_total - bp.kb * gpb);
        if (i % kIssuers != qi) {
          gidx += ng;
          continue;
        }
        const int s = i % NA, sx = i % NX;
        if (!mbar_wait(&afull[s], (i / NA) & 1, a_err, DEVERR_WAIT_MMA)) {
          ok = false;
          break;
        }
        // block i's A slot held block i - NA before: that block's MMAs are done (the unpack team
        // waited for them), so the tile slot of block i + NA (= block i - NA's) is free
        while (ix < nblk && ix <= i + NA) request_tile();
        if (!mbar_wait(&xfull[sx], (i / NX) & 1, a_err, DEVERR_WAIT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t xdesc = xdesc0 + static_cast<uint64_t>((sx * C::kXTile) >> 4);
        const uint32_t a_col = tmem + colA + s * C::kACols;
        for (int gi = 0; gi < ng; ++gi, ++gidx) {
          const int bt = gidx / NBATCH;
          commit_before(bt);
          acquire(bt);
          if (!ok) break;
          const uint32_t d = tmem + colAcc + (bt % NBUF) * (NBATCH * kDN) + (gidx % NBATCH) * kDN;
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
        }
        if (!ok) break;
        tc_commit(&mdone[s]);
      }
      commit_before(nbatch);
      // tiles still in flight after a wait ran out must land before the CTA exits
      for (int j = ix - kIssuers; j >= 0 && j >= ix - NX; j -= kIssuers)
        mbar_wait_for(&xfull[j % NX], static_cast<uint32_t>((j / NX) & 1), nullptr, 0, kDrainLimitNs);
      tc_commit(done);
      mbar_wait(done, 0, a_err, DEVERR_WAIT_TEARDOWN);
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ unpack into TMEM
    // Two teams of four warps (one per TMEM lane quarter) take alternate blocks; each thread
    // unpacks one full row of the block. Only this kernel's shared memory is read: no wait for
    // the previous grid.
    const int q4 = warp & 3, team = (warp - 4) >> 2;
    const int r = 32 * q4 + lane;  // block row = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * q4) << 16;
    for (int i = team; i < nblk; i += 2) {
      const int sw = i % NW, s = i % NA;
      if (!mbar_wait(&wfull[sw], (i / NW) & 1, a_err, DEVERR_WAIT_UNPACK) ||
          !mbar_wait(&mdone[s], ((i / NA) & 1) ^ 1, a_err, DEVERR_WAIT_UNPACK))
        break;
      tc_fence_after();
      const uint32_t ta = tmem + lane_base + colA + s * C::kACols;
      unpack_half_row<I8, BITS>(wring + sw * C::kWBlock, r, 0, ta);
      unpack_half_row<I8, BITS>(wring + sw * C::kWBlock, r, 1, ta + C::kACols / 2);
      // the packed block's values are in registers, handed to the tcgen05.st above: free its slot now
      __syncwarp();
      if (lane == 0) mbar_arrive(&wempty[sw]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[s]);
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ epilogue, one output row per thread
    // Control flow follows the group schedule only; after a wait ran out, `ok` turns off every
    // later wait and TMEM access, and the named barriers are still reached by all four warps.
    grid_dep_wait();
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;
    const int et = threadIdx.x - 384;  // 0..127
    const uint32_t lane_base = static_cast<uint32_t>(32 * q4) << 16;
    const int T = a.T;

    // adapter terms of the tiles whose first block this CTA streams, computed while the pipeline
    // fills (any CTA's fix-up of such a tile reads them only after this CTA has published its
    // segment of the tile); U_cat is staged as fp32 first
    if (a.su_sorted) {
      const int nv = kDN * a.R_pad / 8;  // 8 halves per vector; R_pad is a multiple of 8
      for (int v = et; v < nv; v += 128) {
        const int p = (v * 8) / a.R_pad, j = v * 8 - p * a.R_pad;
        float4 lo = make_float4(0.0f, 0.0f, 0.0f, 0.0f), hi = lo;
        if (p < T) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(a.ucat + static_cast<size_t>(p) * a.R_pad + j));
          const __half2* h = reinterpret_cast<const __half2*>(&u);
          const float2 f0 = __half22float2(h[0]), f1 = __half22float2(h[1]), f2 = __half22float2(h[2]),
                       f3 = __half22float2(h[3]);
          lo = make_float4(f0.x, f0.y, f1.x, f1.y);
          hi = make_float4(f2.x, f2.y, f3.x, f3.y);
        }
        *reinterpret_cast<float4*>(u_s + v * 8) = lo;
        *reinterpret_cast<float4*>(u_s + v * 8 + 4) = hi;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      const int nt_a0 = static_cast<int>((b0 + a.KB - 1) / a.KB), nt_a1 = static_cast<int>((b1 - 1) / a.KB);
      for (int nt = nt_a0; nt <= nt_a1; ++nt) adapter_row(a, u_s, nt, r);
    }

    bool ok = true;
    float acc[kDN];
#pragma unroll
    for (int p = 0; p < kDN; ++p) acc[p] = 0.0f;
    int cur_nt = -1;

    // End of a segment of tile nt: a tile held by this CTA alone is written at once; otherwise the
    // partial goes to its slot and the last CTA to finish the tile adds the partials in segment order.
    auto finish_segment = [&](int nt) {
      const int64_t f0 = static_cast<int64_t>(nt) * a.KB;
      const int c_first = cta_of(f0, a.NB, G);
      const int nseg = cta_of(f0 + a.KB - 1, a.NB, G) - c_first + 1;
      const int seg = c - c_first;
      const int o = nt * kTileN + r;
      const size_t tile_row = (static_cast<size_t>(nt) * kTileN + r) * kDN;
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

    // group scales, one per group and row, copied by the thread itself (cp.async) into its own
    // column of a four-batch ring: batch bt + 3 is requested when batch bt starts. An fp16 scale
    // travels in the aligned 4-byte pair that holds it.
    GroupPos pf;
    pf.init(pos0, gpb, a.G_total);
    int pf_left = ngroups;
    const size_t sc_total = static_cast<size_t>(a.G_total) * a.N;
    auto request_batch_scales = [&](int bt) {
      uint32_t* dst = sc_s + (bt % C::kScaleBatches) * NBATCH * kTileN + et;
      for (int k = 0; k < NBATCH && pf_left > 0; ++k, --pf_left, pf.next(a.KB, gpb, a.G_total)) {
        const int o = pf.bp.nt * kTileN + r;
        if (o >= a.N) continue;
        const size_t idx = static_cast<size_t>(pf.bp.kb * gpb + pf.gi) * a.N + o;
        if (a.sw_f16) {
          const size_t e0 = idx & ~size_t(1);
          cp_async4_n(dst + k * kTileN, reinterpret_cast<const unsigned short*>(a.w_scale) + e0,
                      (e0 + 1 < sc_total) ? 4u : 2u);
        } else {
          cp_async4_n(dst + k * kTileN, a.w_scale + idx, 4u);
        }
      }
      cp_async_commit();
    };
    // the scale of group k of batch bt (j = its group index in the weight's group order, o its row)
    auto scale_of = [&](int bt, int k, int j, int o) -> float {
      const uint32_t w = sc_s[((bt % C::kScaleBatches) * NBATCH + k) * kTileN + et];
      if (a.sw_f16) {
        const bool high = ((static_cast<int64_t>(j) * a.N + o) & 1) != 0;
        const unsigned short h = static_cast<unsigned short>(high ? (w >> 16) : (w & 0xFFFFu));
        float f;
        asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"(h));
        return f;
      }
      return __uint_as_float(w);
    };
    for (int b = 0; b < C::kScaleBatches - 1; ++b) request_batch_scales(b);

    // a new tile starts in the group sequence: finish the previous one
    auto enter_tile = [&](int nt) {
      if (cur_nt >= 0) finish_segment(cur_nt);
      cur_nt = nt;
#pragma unroll
      for (int p = 0; p < kDN; ++p) acc[p] = 0.0f;
    };

    GroupPos gp;
    gp.init(pos0, gpb, a.G_total);
    int gleft = ngroups;
    for (int bt = 0; bt < nbatch; ++bt) {
      request_batch_scales(bt + C::kScaleBatches - 1);
      cp_async_wait_group<C::kScaleBatches - 1>();  // batch bt's scales have landed (this thread's own copies)
      const int buf = bt % NBUF;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&accf[buf], (bt / NBUF) & 1, a_err, DEVERR_WAIT_EPILOGUE));
      if (ok) tc_fence_after();
      const int nb = min(NBATCH, gleft);
      gleft -= nb;
      const uint32_t bcol = tmem + lane_base + colAcc + buf * (NBATCH * kDN);
      if (gp.bp.nt != cur_nt) enter_tile(gp.bp.nt);
      const int j0 = gp.bp.kb * gpb + gp.gi;
      if (ok && nb == NBATCH && nb <= a.G_total - j0 && !a.dbg_acc) {
        // the whole batch lies in the current tile: its groups are consecutive in the weight's
        // group order (j0 .. j0 + 7), read two at a time
        const int o = cur_nt * kTileN + r;
#pragma unroll
        for (int h = 0; h < NBATCH / 2; ++h) {
          uint32_t v[2 * kDN];
          tmem_ld32(bcol + h * 2 * kDN, v);
          tmem_wait_ld();
          reg_fence(v);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const float sw = scale_of(bt, 2 * h + k, j0 + 2 * h + k, o);
            if constexpr (I8) {
              const float swq = sw * 0.0625f;  // codes entered the MMA as 16*q
#pragma unroll
              for (int p = 0; p < kDN; ++p)
                acc[p] = fmaf(static_cast<float>(static_cast<int32_t>(v[k * kDN + p])), swq, acc[p]);
            } else {
#pragma unroll
              for (int p = 0; p < kDN; ++p) acc[p] = fmaf(__uint_as_float(v[k * kDN + p]), sw, acc[p]);
            }
          }
        }
#pragma unroll
        for (int k = 0; k < NBATCH; ++k) gp.next(a.KB, gpb, a.G_total);
      } else {
        for (int k = 0; k < nb; ++k, gp.next(a.KB, gpb, a.G_total)) {
          const int nt = gp.bp.nt;
          if (nt != cur_nt) enter_tile(nt);
          if (!ok) continue;
          uint32_t v[kDN];
          tmem_ld16(bcol + k * kDN, v);
          tmem_wait_ld();
          reg_fence(v);
          const int j = gp.bp.kb * gpb + gp.gi, o = nt * kTileN + r;
          const float sw = (o < a.N) ? scale_of(bt, k, j, o) : 0.0f;
          if constexpr (I8) {
            const float swq = sw * 0.0625f;  // codes entered the MMA as 16*q
#pragma unroll
            for (int p = 0; p < kDN; ++p) acc[p] = fmaf(static_cast<float>(static_cast<int32_t>(v[p])), swq, acc[p]);
            if (a.dbg_acc && o < a.N) {
#pragma unroll
              for (int p = 0; p < kDN; ++p) {
                if (p >= T) break;
                a.dbg_acc[(static_cast<size_t>(__ldg(a.perm + p)) * a.N + o) * a.G_total + j] =
                    static_cast<int32_t>(v[p]) / 16;
              }
            }
          } else {
#pragma unroll
            for (int p = 0; p < kDN; ++p) acc[p] = fmaf(__uint_as_float(v[p]), sw, acc[p]);
          }
        }
      }
      // the batch's sums are in registers: the buffer can take batch bt + NBUF
      if (ok) tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&acce[buf]);
    }
    if (cur_nt >= 0) finish_segment(cur_nt);
    cp_async_wait_group<0>();
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
  if (q.T > kDN || q.T < 1 || R_pad > kMaxRpad || R_pad % 8 != 0) return cudaErrorInvalidValue;
  if (int8) {
    if (w_bits != 4) return cudaErrorInvalidValue;
    return launch_qdec_t<true, 4>(tm_x, a, plan.grid, st);
  }
  if (w_bits == 4) return launch_qdec_t<false, 4>(tm_x, a, plan.grid, st);
  if (w_bits == 3) return launch_qdec_t<false, 3>(tm_x, a, plan.grid, st);
  return cudaErrorInvalidValue;
}

}  // namespace qe
