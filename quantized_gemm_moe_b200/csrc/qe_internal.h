// Internal declarations shared by the host API (qe_api.cu) and the kernel files.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace qe {

constexpr int kTileN = 128;       // output rows per weight block / GEMM tile (MMA M)
constexpr int kTileK = 128;       // input channels per weight block / pipeline stage
constexpr int kW4BlockBytes = 8192;
constexpr int kW3BlockBytes = 6144;
constexpr int kMaxRouted = 16;
constexpr int kAdapterAtom = 64;  // bf16 elements per 128-byte swizzle row

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }
inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Packed adapter buffer geometry.
//   A_catT [R_tot][K] bf16: the rows of the adapter/router GEMM. Rows [0, r_s) are the shared
//     down-projection. Dense routed experts add rows [r_s, R_a) (A_r[e] columns expert by
//     expert) and the router G (transposed) sits at rows [R_rt, R_rt + N_r) with R_rt = R_pad.
//     Cluster-sparse routed experts (kc > 0) have no GEMM rows: the router follows the shared
//     rows (R_rt = the smallest supported GEMM width >= round_up(r_s, 16) + 16, minus 16).
//     All other rows are zero. One GEMM gives U and the router logits.
//   B_catT [N][R_pad] fp16: the up-projections of the shared and all routed columns.
//   kc > 0: the channels of each expert, int32 [N_r][kc], and its down-projection over them,
//     bf16 [N_r][kc][r_r].
struct AdapterGeom {
  int r_s, n_r, r_r;
  int R_a;    // r_s + n_r * r_r
  int R_pad;  // round_up(R_a, 64), or 0 when the layer has no adapters
  int R_tot;  // rows of A_catT = columns of the adapter/router GEMM
  int R_rt;   // first router row
  int kc;     // channels per routed expert (0: dense routed experts)
  size_t off_acat, off_bcat, off_rch, off_rar, bytes;
};
inline int sparse_gemm_width(int r_s) {
  // adapter/router GEMM widths the library instantiates (see launch_ugemm)
  const int need = static_cast<int>(round_up(r_s, 16)) + 16;
  const int widths[] = {16, 32, 48, 64, 80, 128, 144, 192, 208, 256};
  for (int w : widths)
    if (w >= need) return w;
  return 0;
}
inline AdapterGeom adapter_geom(int K, int N, int r_s, int n_r, int r_r, int kc) {
  AdapterGeom g;
  g.r_s = r_s;
  g.n_r = n_r;
  g.r_r = r_r;
  g.kc = (r_r > 0) ? kc : 0;
  g.R_a = r_s + n_r * r_r;
  g.R_pad = g.R_a > 0 ? static_cast<int>(round_up(g.R_a, kAdapterAtom)) : 0;
  if (g.kc == 0) {
    g.R_tot = (g.R_pad + 16 <= 256) ? g.R_pad + 16 : g.R_pad + 64;
    g.R_rt = g.R_pad;
  } else {
    g.R_tot = sparse_gemm_width(r_s);
    g.R_rt = g.R_tot - 16;
  }
  g.off_acat = 0;
  g.off_bcat = align256(g.off_acat + size_t(g.R_tot) * K * 2);
  g.off_rch = align256(g.off_bcat + size_t(N) * g.R_pad * 2);
  g.off_rar = align256(g.off_rch + size_t(n_r) * g.kc * 4);
  g.bytes = align256(g.off_rar + size_t(n_r) * g.kc * (g.kc ? r_r : 0) * 2);
  return g;
}

// ------------------------------------------------------------------ kernel launchers
// Each returns the launch's cudaError_t. The host API validates before calling.

// w_scale: fp32 [G][N], or fp16 when s16 != 0 (a scale beyond fp16 is saturated, device error 0x203).
cudaError_t launch_quantize_weights(const void* W, bool w_bf16, const float* s, int N, int K, int group,
                                    int w_bits, uint8_t* packed, void* w_scale, int s16, int* err,
                                    cudaStream_t st);
cudaError_t launch_colstats(const void* W, bool w_bf16, int N, int K, float* w_mean, float* w_colmax,
                            cudaStream_t st);
// s_inv[k] = fl32(1/s[k]) (IEEE division).
cudaError_t launch_recip(const float* s, int K, float* s_inv, cudaStream_t st);
cudaError_t launch_unpack_weights(const uint8_t* packed, int N, int K, int w_bits, int8_t* codes,
                                  cudaStream_t st);
cudaError_t launch_pack_adapters(const AdapterGeom& g, int K, int N, const uint16_t* A_s, const uint16_t* B_s,
                                 const uint16_t* A_r, const uint16_t* B_r, const uint16_t* G, const int32_t* channels,
                                 uint8_t* out, int* err, cudaStream_t st);

// Router logits + argmin, and (when sa != nullptr) the per-token absmax -> scale, on CUDA cores
// (the standalone router entry point and the activation-quantization diagnostic).
cudaError_t launch_route_stats(const void* X, bool x_bf16, const float* s_inv, const uint16_t* G, int T, int K,
                               int n_r, int qmax, int32_t* expert, float* sa, float* logits, cudaStream_t st);
// Stable bucket sort of tokens by expert: perm (sorted pos -> token), pos (token -> sorted pos), offsets.
cudaError_t launch_bucket(const int32_t* expert, int T, int n_r, int32_t* perm, int32_t* pos, int32_t* offsets,
                          cudaStream_t st);
// Per-token quantization of x*s_inv with the scale sa_tok[t], written at row pos[t] (pos == nullptr: row t).
//   codes != nullptr: int8 codes, sa_sorted[pos] = sa_tok[t]
//   act16 != nullptr: bf16(x*s_inv) (weight-only layers)
// (used by the activation-quantization diagnostic entry point)
cudaError_t launch_act_quant(const void* X, bool x_bf16, const float* s_inv, int T, int K, int qmax,
                             const float* sa_tok, const int32_t* pos, int8_t* codes, float* sa_sorted,
                             uint16_t* act16, uint16_t* xb16, uint16_t* xlo16, cudaStream_t st);

// fp32 inputs: x = hi + lo (both bf16, token order) for the bf16 tensor-core GEMM, and the
// per-token absmax of fl32(x*s_inv) (one slot).
cudaError_t launch_split_f32(const float* X, const float* s_inv, int T, int K, uint16_t* xhi, uint16_t* xlo,
                             float* amax, cudaStream_t st);

// P[slot][t][c] = sum over this split's K range of X[t][k] * A_catT[c][k], c < R_tot (tcgen05, bf16):
// the adapter down-projections and, in columns [R_pad, R_pad + N_r), the router logits.
struct UgemmPlan {
  int splits;
  int kchunks_per_split;  // 64-wide K chunks per split
  int nu;                 // N tile (columns of A_catT per CTA), <= 256
  int ntiles;
};
UgemmPlan plan_ugemm(int T, int K, int R_tot);
// zero_ctr != nullptr: the first CTA also sets *zero_ctr = 0 (the route/quant launch's barrier).
cudaError_t launch_ugemm(const CUtensorMap& tm_x, const CUtensorMap& tm_acat, const UgemmPlan& plan, int T,
                         int K, int R_tot, float* partial, unsigned* zero_ctr, int* err, cudaStream_t st);
// Routing, stable bucket sort and activation quantization in one cooperative launch (grid barrier
// between the per-token routing and the sort). route: expert = argmin of the router logits (sum of
// the U partial slots, columns [R_pad, R_pad+N_r)), sa_tok = absmax/qmax (absmax from X for bf16
// inputs, amax[t] for fp32 inputs; sa_tok == nullptr for weight-only layers), perm/pos/offsets.
// quant: codes (or bf16 act16) at row pos[t], sa_sorted, and U_cat / su_sorted.
// *barrier must be 0 when the launch starts.
constexpr int kRouteQuantMaxGrid = 1024;
constexpr int kMaxForwardDin = 32768;  // the route/quant launch keeps s_inv in shared memory
struct RouteQuantParams {
  const float* partial;
  int nslots, R_tot, R_pad, R_rt, n_r, r_s, r_r, R_a;
  // cluster-sparse routed experts (kc > 0): expert e's routed U columns are
  // sum_i x[t][rch[e][i]] * rar[e][i][j] (raw x), not GEMM columns
  int kc;
  const int32_t* rch;
  const uint16_t* rar;
  const void* X;
  bool x_bf16;
  const float* s_inv;
  const float* amax;
  int T, K, qmax;
  int do_route, do_quant;
  int32_t* expert;
  float* sa_tok;
  int32_t* perm;
  int32_t* pos;
  int32_t* offsets;
  int32_t* counts;  // [kRouteQuantMaxGrid][kMaxRouted]
  unsigned* barrier;
  int8_t* codes;
  uint16_t* act16;
  float* sa_sorted;
  uint16_t* ucat;
  float* su_sorted;
  unsigned* zero_words;  // cleared by the launch (the decode product's tile counters), may be null
  int n_zero_words;
  int* err;
};
cudaError_t launch_route_quant(const RouteQuantParams& q, cudaStream_t st);

// Main quantized GEMM (W4 x A8/A6 codes, tcgen05 kind::i8) with per-group promotion,
// per-token scale, adapter MMA in the epilogue and scatter to token order.
struct QgemmArgs {
  const uint8_t* w_packed;
  const float* w_scale;     // [G][N] fp32, or fp16 when sw_f16
  int sw_f16;
  const float* sa_sorted;   // [T]
  const float* su_sorted;   // [T] adapter scale of U_cat rows
  const int32_t* perm;      // [T]
  int T, N, K, group;
  int KB;                   // ceil(K / 128)
  int adapter_atoms;        // R_pad / 64, or 0 when the layer has no adapters
  int splits, kb_per_split;
  void* Y;                  // [T][N] (splits == 1)
  int y_bf16;
  float* partial;           // [splits][T][N] sorted rows (splits > 1)
  int32_t* dbg_acc;         // [T][N][G] token order, or nullptr
  int* err;                 // device error word
};
int pick_qgemm_bn(int T, int N, int K, int* splits_out, int* kbps_out);
cudaError_t launch_qgemm(int BN, const CUtensorMap& tm_xq, const CUtensorMap& tm_bcat, const CUtensorMap& tm_ucat,
                         const QgemmArgs& a, cudaStream_t st);
cudaError_t launch_splitk_reduce(const float* partial, int splits, const int32_t* perm, int T, int N, void* Y,
                                 int y_bf16, cudaStream_t st);

// Product of a decode-sized batch (T <= 16): every (output tile, K block) split evenly over the
// SMs, weights unpacked into TMEM as the MMA's A operand, per-tile fix-up of the segment partials
// in a fixed order. int8 = W4 x A8/A6 codes (kind::i8); otherwise bf16 activations against W4/W3
// weights (kind::f16). part/ad/cnt live in the workspace; cnt must be zero at launch (the
// route/quantize launch clears it, and each launch leaves it zero).
struct DecodePlan {
  int NT, KB, grid, maxseg;
  int64_t NB;
  size_t part_bytes, ad_bytes;
  int cnt_words;
};
DecodePlan plan_decode(int N, int K, int n_sm);
int decode_grid_sms();  // SMs of the current device (0 when there is none)
cudaError_t launch_qdec(int w_bits, bool int8, const CUtensorMap& tm_x, const DecodePlan& plan, const QgemmArgs& q,
                        const uint16_t* ucat, const uint16_t* bcat, int R_pad, float* part, float* ad,
                        unsigned* cnt, cudaStream_t st);
constexpr int kDecodeMaxT = 16;
constexpr int kDecodeMaxRpad = 384;  // the decode product stages U_cat in shared memory

// Weight-only (W3A16 / W4A16) product on the tensor cores: codes unpacked to bf16, bf16
// activations (act16, bucket order), per-group fp32 sums scaled by sw, adapter epilogue.
int pick_wgemm_bn(int T, int N, int K, int* splits_out, int* kbps_out);
cudaError_t launch_wgemm(int bits, int BN, const CUtensorMap& tm_act, const CUtensorMap& tm_bcat,
                         const CUtensorMap& tm_ucat, const QgemmArgs& a, cudaStream_t st);

// Positions of the token-dependent channels (histogram rank k .. k+C-1), -1 elsewhere.
cudaError_t launch_split_channels(const int32_t* hist, int d, int k, int C, int32_t* pos, cudaStream_t st);

// Co-occurrence counts O [C][C] of the token-dependent channels in each token's Top-k set, and
// their NPMI S (optional). O is zeroed here.
cudaError_t launch_cooc_npmi(const int32_t* idx, int T, int k, const int32_t* pos, int d_in, int C, int32_t* O,
                             float* S, float threshold, cudaStream_t st);

// One CTA whose single wait runs out after limit_ns (the bounded-wait self-test).
cudaError_t launch_wait_selftest(int* err, uint64_t limit_ns, cudaStream_t st);

// Device error word (one per device, in the library's own device memory).
int* device_error_ptr();  // nullptr when the symbol lookup fails
// The calling thread's current CUDA context (CUcontext), or nullptr; keys the per-device
// caches of device symbol addresses.
void* current_context();
cudaError_t read_device_error(int* value, bool clear, cudaStream_t st);

// Top-k importance. bf16 rows with 7680 <= K <= 30720 take the streaming kernel (one CTA per
// SM, rows staged by bulk copies); others, and rows it leaves unresolved, the radix-select kernel.
cudaError_t launch_topk(const void* X, bool x_bf16, const float* w_mean, int T, int K, int k, int32_t* idx,
                        int32_t* hist, int* err, cudaStream_t st);

}  // namespace qe
