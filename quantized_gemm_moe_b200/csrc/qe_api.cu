// Host side of the C ABI declared in include/qe.h: argument validation,
// workspace planning, TMA tensor-map encoding and the launch sequence of the
// QE linear layer. Nothing here allocates device memory.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/qe.h"
#include "qe_internal.h"

namespace qe {
namespace {

thread_local char g_last_cuda_error[256] = "";

qe_status cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", where, cudaGetErrorString(e));
  return QE_ERR_CUDA;
}

#define QE_CUDA(call, where)                          \
  do {                                                \
    cudaError_t e_ = (call);                          \
    if (e_ != cudaSuccess) return cuda_fail(e_, where); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

qe_status check_desc(const qe_layer_desc* d) {
  if (!d) return QE_ERR_INVALID_ARG;
  if (d->d_in <= 0 || d->d_out <= 0 || d->group <= 0) return QE_ERR_INVALID_ARG;
  if (d->group != 64 && d->group != 128) return QE_ERR_UNSUPPORTED;
  if (d->d_in % d->group != 0) return QE_ERR_INVALID_ARG;
  if (d->d_in < 128) return QE_ERR_UNSUPPORTED;
  if (d->w_bits != 3 && d->w_bits != 4) return QE_ERR_UNSUPPORTED;
  if (d->a_bits != 6 && d->a_bits != 8 && d->a_bits != 16) return QE_ERR_UNSUPPORTED;
  if (d->a_bits != 16 && d->w_bits != 4) return QE_ERR_UNSUPPORTED;  // W3 runs weight-only
  if (d->n_routed < 1 || d->n_routed > kMaxRouted) return QE_ERR_UNSUPPORTED;
  if (d->rank_shared < 0 || d->rank_routed < 0) return QE_ERR_INVALID_ARG;
  if (d->rank_shared + int64_t(d->n_routed) * d->rank_routed > 512) return QE_ERR_UNSUPPORTED;
  if (d->d_in > (1 << 24) || d->d_out > (1 << 24)) return QE_ERR_UNSUPPORTED;
  if (d->routed_channels < 0 || d->routed_channels > d->d_in) return QE_ERR_INVALID_ARG;
  if (d->routed_channels > 0 && (d->rank_routed == 0 || sparse_gemm_width(d->rank_shared) == 0))
    return QE_ERR_UNSUPPORTED;
  if (d->w_scale_fp16 != 0 && d->w_scale_fp16 != 1) return QE_ERR_INVALID_ARG;
  return QE_OK;
}

int qmax_of(int bits) { return (1 << (bits - 1)) - 1; }

size_t packed_bytes(const qe_layer_desc* d) {
  const size_t blocks = size_t(ceil_div(d->d_out, kTileN)) * size_t(ceil_div(d->d_in, kTileK));
  return blocks * (d->w_bits == 4 ? kW4BlockBytes : kW3BlockBytes);
}

AdapterGeom geom_of(const qe_layer_desc* d) {
  return adapter_geom(d->d_in, d->d_out, d->rank_shared, d->n_routed, d->rank_routed, d->routed_channels);
}

// ------------------------------------------------------------------ workspace plan
struct Plan {
  int T, K, N;
  bool has_ad;
  AdapterGeom g;
  UgemmPlan up;
  int bn, msplits, kbps;  // main product
  int uslots;             // GEMM partial slots: splits, doubled for fp32 inputs (hi and lo passes)
  bool dec;               // T <= 16: the decode product (stream-K over the SMs, in-kernel fix-up)
  DecodePlan dp;
  size_t off_expert, off_perm, off_pos, off_offsets, off_sa_tok, off_sa_sorted, off_su_sorted, off_act, off_xhi,
      off_xlo, off_amax, off_upart, off_ucat, off_ypart, off_counts, off_barrier, off_dpart, off_dad, off_dcnt,
      bytes;
};

Plan make_plan(const qe_layer_desc* d, int T, bool x_bf16) {
  Plan p{};
  p.T = T;
  p.K = d->d_in;
  p.N = d->d_out;
  p.g = geom_of(d);
  p.has_ad = p.g.R_a > 0;
  const int Tm = std::max(T, 1);
  p.up = plan_ugemm(Tm, p.K, p.g.R_tot);
  p.dec = Tm <= kDecodeMaxT && (!p.has_ad || p.g.R_pad <= kDecodeMaxRpad);
  if (p.dec) {
    p.dp = plan_decode(p.N, p.K, decode_grid_sms());
    p.bn = 16;
    p.msplits = 1;
    p.kbps = static_cast<int>(ceil_div(p.K, kTileK));
  } else if (d->a_bits == 16) {
    p.bn = pick_wgemm_bn(Tm, p.N, p.K, &p.msplits, &p.kbps);
  } else {
    p.bn = pick_qgemm_bn(Tm, p.N, p.K, &p.msplits, &p.kbps);
  }
  p.uslots = p.up.splits * (x_bf16 ? 1 : 2);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  p.off_expert = take(size_t(Tm) * 4);
  p.off_perm = take(size_t(Tm) * 4);
  p.off_pos = take(size_t(Tm) * 4);
  p.off_offsets = take(size_t(kMaxRouted + 1) * 4);
  p.off_sa_tok = take(size_t(Tm) * 4);
  p.off_sa_sorted = take(size_t(Tm) * 4);
  p.off_su_sorted = take(size_t(Tm) * 4);
  p.off_act = take(size_t(Tm) * p.K * (d->a_bits == 16 ? 2 : 1));
  p.off_xhi = x_bf16 ? 0 : take(size_t(Tm) * p.K * 2);
  p.off_xlo = x_bf16 ? 0 : take(size_t(Tm) * p.K * 2);
  p.off_amax = x_bf16 ? 0 : take(size_t(Tm) * 4);
  p.off_upart = take(size_t(p.uslots) * Tm * p.g.R_tot * 4);
  p.off_ucat = p.has_ad ? take(size_t(Tm) * p.g.R_pad * 2) : 0;
  p.off_ypart = (p.msplits > 1) ? take(size_t(p.msplits) * Tm * p.N * 4) : 0;
  p.off_counts = take(size_t(kRouteQuantMaxGrid) * kMaxRouted * 4);
  p.off_barrier = take(4);
  if (p.dec) {
    p.off_dpart = take(p.dp.part_bytes);
    p.off_dad = take(p.dp.ad_bytes);
    p.off_dcnt = take(size_t(p.dp.cnt_words) * 4);
  }
  p.bytes = o;
  return p;
}

// ------------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 2-D row-major [rows][cols] tensor, box {box_cols, box_rows}, 128-byte swizzle, zero fill out of bounds.
qe_status make_tmap(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t cols,
                    uint64_t rows, uint32_t box_cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) {
    snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled unavailable");
    return QE_ERR_CUDA;
  }
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * elem_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled failed (%d)", int(r));
    return QE_ERR_CUDA;
  }
  return QE_OK;
}

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// Every check of a forward call that does not depend on the workspace, in the order the
// header documents them. Both forward entry points run it before they size any scratch.
// T == 0 passes (the caller returns QE_OK without launching anything).
qe_status check_forward_args(const qe_layer_desc* d, const qe_layer_weights* w, const void* X, qe_dtype xd,
                             int32_t T, const void* Y, qe_dtype yd) {
  qe_status s = check_desc(d);
  if (s != QE_OK) return s;
  if (!w || !w->w_packed || !w->w_scale || !w->s_inv || !w->adapters) return QE_ERR_INVALID_ARG;
  if (T < 0 || T > (1 << 20)) return QE_ERR_INVALID_ARG;
  if (d->d_in > kMaxForwardDin) return QE_ERR_UNSUPPORTED;
  if (xd != QE_F32 && xd != QE_BF16) return QE_ERR_INVALID_ARG;
  if (yd != QE_F32 && yd != QE_BF16) return QE_ERR_INVALID_ARG;
  if (T == 0) return QE_OK;
  if (!X || !Y) return QE_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Y) || !aligned16(w->w_packed) || !aligned16(w->w_scale) ||
      !aligned16(w->s_inv) || !aligned16(w->adapters))
    return QE_ERR_ALIGNMENT;
  return QE_OK;
}

qe_status forward_impl(const qe_layer_desc* d, const qe_layer_weights* w, const void* X, qe_dtype xd, int32_t T,
                       void* Y, qe_dtype yd, void* ws, size_t ws_bytes, int32_t* dbg_acc, int32_t* dbg_expert,
                       int32_t* dbg_perm, float* dbg_sa, int32_t stages, cudaStream_t st) {
  qe_status s = check_forward_args(d, w, X, xd, T, Y, yd);
  if (s != QE_OK || T == 0) return s;
  const bool x_bf16 = xd == QE_BF16;
  const Plan p = make_plan(d, T, x_bf16);
  if (!ws || ws_bytes < p.bytes) return QE_ERR_WORKSPACE;
  if (!aligned16(ws)) return QE_ERR_ALIGNMENT;
  int* err = device_error_ptr();
  const uint8_t* ad = static_cast<const uint8_t*>(w->adapters);
  const uint16_t* acat = reinterpret_cast<const uint16_t*>(ad + p.g.off_acat);
  const uint16_t* bcat = reinterpret_cast<const uint16_t*>(ad + p.g.off_bcat);
  int32_t* expert = at<int32_t>(ws, p.off_expert);
  int32_t* perm = at<int32_t>(ws, p.off_perm);
  int32_t* pos = at<int32_t>(ws, p.off_pos);
  int32_t* offsets = at<int32_t>(ws, p.off_offsets);
  float* sa_tok = at<float>(ws, p.off_sa_tok);
  float* sa_sorted = at<float>(ws, p.off_sa_sorted);
  float* su_sorted = at<float>(ws, p.off_su_sorted);
  float* amax = x_bf16 ? nullptr : at<float>(ws, p.off_amax);
  float* upart = at<float>(ws, p.off_upart);
  const bool wonly = d->a_bits == 16;
  const int qmax = wonly ? 1 : qmax_of(d->a_bits);
  const int K = p.K, N = p.N;

  unsigned* barrier = at<unsigned>(ws, p.off_barrier);
  int8_t* codes = wonly ? nullptr : at<int8_t>(ws, p.off_act);
  uint16_t* act16 = wonly ? at<uint16_t>(ws, p.off_act) : nullptr;
  uint16_t* ucat = p.has_ad ? at<uint16_t>(ws, p.off_ucat) : nullptr;

  // 1. one tensor-core GEMM: adapter down-projections + router logits
  //    (its first CTA also clears the grid barrier of step 2)
  const bool project = (stages & QE_STAGE_PROJECT) != 0;
  const bool route = (stages & QE_STAGE_ROUTE) != 0, quant = (stages & QE_STAGE_QUANT) != 0;
  if (project) {
    CUtensorMap tm_acat;
    if ((s = make_tmap(&tm_acat, acat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, p.g.R_tot, kAdapterAtom, p.up.nu)) !=
        QE_OK)
      return s;
    if (x_bf16) {
      CUtensorMap tm_x;
      if ((s = make_tmap(&tm_x, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, T, kAdapterAtom, 128)) != QE_OK) return s;
      QE_CUDA(launch_ugemm(tm_x, tm_acat, p.up, T, K, p.g.R_tot, upart, barrier, err, st), "ugemm");
    } else {
      // fp32 input: x = hi + lo in bf16, two passes into consecutive partial slots
      uint16_t* xhi = at<uint16_t>(ws, p.off_xhi);
      uint16_t* xlo = at<uint16_t>(ws, p.off_xlo);
      QE_CUDA(launch_split_f32(static_cast<const float*>(X), w->s_inv, T, K, xhi, xlo, amax, st), "split_f32");
      CUtensorMap tm_hi, tm_lo;
      if ((s = make_tmap(&tm_hi, xhi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, T, kAdapterAtom, 128)) != QE_OK) return s;
      if ((s = make_tmap(&tm_lo, xlo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, T, kAdapterAtom, 128)) != QE_OK) return s;
      QE_CUDA(launch_ugemm(tm_hi, tm_acat, p.up, T, K, p.g.R_tot, upart, barrier, err, st), "ugemm_hi");
      QE_CUDA(launch_ugemm(tm_lo, tm_acat, p.up, T, K, p.g.R_tot, upart + size_t(p.up.splits) * T * p.g.R_tot,
                           nullptr, err, st),
              "ugemm_lo");
    }
  }
  // 2. argmin routing, per-token absmax and scale, stable bucket sort, then quantization in bucket
  //    order and the expert-masked adapter rows U_cat: one cooperative launch
  if (route || quant) {
    if (route && !project) QE_CUDA(cudaMemsetAsync(barrier, 0, 4, st), "memset");
    RouteQuantParams q{};
    q.partial = upart;
    q.nslots = p.uslots;
    q.R_tot = p.g.R_tot;
    q.R_pad = p.g.R_pad;
    q.R_rt = p.g.R_rt;
    q.kc = p.g.kc;
    q.rch = reinterpret_cast<const int32_t*>(static_cast<const uint8_t*>(w->adapters) + p.g.off_rch);
    q.rar = reinterpret_cast<const uint16_t*>(static_cast<const uint8_t*>(w->adapters) + p.g.off_rar);
    q.n_r = d->n_routed;
    q.r_s = d->rank_shared;
    q.r_r = d->rank_routed;
    q.R_a = p.g.R_a;
    q.X = X;
    q.x_bf16 = x_bf16;
    q.s_inv = w->s_inv;
    q.amax = amax;
    q.T = T;
    q.K = K;
    q.qmax = qmax;
    q.do_route = route;
    q.do_quant = quant;
    q.expert = expert;
    q.sa_tok = wonly ? nullptr : sa_tok;
    q.perm = perm;
    q.pos = pos;
    q.offsets = offsets;
    q.counts = at<int32_t>(ws, p.off_counts);
    q.barrier = barrier;
    q.codes = codes;
    q.act16 = act16;
    q.sa_sorted = sa_sorted;
    q.ucat = ucat;
    q.su_sorted = su_sorted;
    q.zero_words = p.dec ? at<unsigned>(ws, p.off_dcnt) : nullptr;
    q.n_zero_words = p.dec ? p.dp.cnt_words : 0;
    q.err = err;
    QE_CUDA(launch_route_quant(q, st), "route_quant");
  }
  // 5. main product
  if (!(stages & QE_STAGE_PRODUCT)) return QE_OK;
  float* ypart = p.msplits > 1 ? at<float>(ws, p.off_ypart) : nullptr;
  const int y_bf16 = yd == QE_BF16;
  {
    CUtensorMap tm_act, tm_bcat, tm_ucat;
    if (wonly) {
      if ((s = make_tmap(&tm_act, act16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, T, 64, p.bn)) != QE_OK) return s;
    } else {
      if ((s = make_tmap(&tm_act, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, T, kTileK, p.bn)) != QE_OK) return s;
    }
    if (p.has_ad) {
      if ((s = make_tmap(&tm_bcat, bcat, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, p.g.R_pad, N, kAdapterAtom, kTileN)) !=
          QE_OK)
        return s;
      if ((s = make_tmap(&tm_ucat, ucat, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, p.g.R_pad, T, kAdapterAtom, p.bn)) !=
          QE_OK)
        return s;
    } else {
      tm_bcat = tm_act;
      tm_ucat = tm_act;
    }
    QgemmArgs a{};
    a.w_packed = static_cast<const uint8_t*>(w->w_packed);
    a.w_scale = w->w_scale;
    a.sw_f16 = d->w_scale_fp16;
    a.sa_sorted = sa_sorted;
    a.su_sorted = p.has_ad ? su_sorted : nullptr;
    a.perm = perm;
    a.T = T;
    a.N = N;
    a.K = K;
    a.group = d->group;
    a.KB = static_cast<int>(ceil_div(K, kTileK));
    a.adapter_atoms = p.has_ad ? p.g.R_pad / kAdapterAtom : 0;
    a.splits = p.msplits;
    a.kb_per_split = p.kbps;
    a.Y = Y;
    a.y_bf16 = y_bf16;
    a.partial = ypart;
    a.dbg_acc = wonly ? nullptr : dbg_acc;
    a.err = err;
    if (p.dec)
      QE_CUDA(launch_qdec(d->w_bits, !wonly, tm_act, p.dp, a, ucat, bcat, p.g.R_pad, at<float>(ws, p.off_dpart),
                          at<float>(ws, p.off_dad), at<unsigned>(ws, p.off_dcnt), st),
              "qdec");
    else if (wonly)
      QE_CUDA(launch_wgemm(d->w_bits, p.bn, tm_act, tm_bcat, tm_ucat, a, st), "wgemm");
    else
      QE_CUDA(launch_qgemm(p.bn, tm_act, tm_bcat, tm_ucat, a, st), "qgemm");
  }
  if (p.msplits > 1) QE_CUDA(launch_splitk_reduce(ypart, p.msplits, perm, T, N, Y, y_bf16, st), "splitk_reduce");
  if (dbg_expert) QE_CUDA(cudaMemcpyAsync(dbg_expert, expert, size_t(T) * 4, cudaMemcpyDeviceToDevice, st), "copy");
  if (dbg_perm) QE_CUDA(cudaMemcpyAsync(dbg_perm, perm, size_t(T) * 4, cudaMemcpyDeviceToDevice, st), "copy");
  if (dbg_sa) QE_CUDA(cudaMemcpyAsync(dbg_sa, sa_tok, size_t(T) * 4, cudaMemcpyDeviceToDevice, st), "copy");
  return QE_OK;
}

// ------------------------------------------------------------------ no-allocation variant
// Scratch for qe_linear_forward_noalloc: a fixed array in the library's own
// device memory, so that caller needs to provide no workspace. It exists on
// every GPU that loads this module and stays until the process exits. All
// calls share it; it keeps the last call's contents (the forward overwrites
// every byte it reads before reading it, so nothing needs clearing).
static __device__ __align__(256) uint8_t g_static_scratch[QE_NOALLOC_WORKSPACE_BYTES];

// Device address of g_static_scratch for the current device. Host code must not use the
// array's name as an address: on the host it is only a stand-in symbol, not device memory.
// The address is looked up once per device and context: if the device's context is replaced
// (after cudaDeviceReset, the module is loaded again), the next call looks it up again.
qe_status static_scratch(void** out) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  static void* ctx_of[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return QE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  void* ctx = current_context();
  if (!addr[dev] || ctx != ctx_of[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    // The lookup can load this module onto the device, and the loader initializes the
    // array asynchronously. Wait for that once, so it cannot overwrite the first call's data.
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize(static scratch set-up)");
    addr[dev] = p;
    ctx_of[dev] = current_context();
  }
  *out = addr[dev];
  return QE_OK;
}

}  // namespace
}  // namespace qe

using namespace qe;

extern "C" {

size_t qe_packed_weight_bytes(const qe_layer_desc* desc) {
  if (check_desc(desc) != QE_OK) return 0;
  return packed_bytes(desc);
}

size_t qe_adapter_packed_bytes(const qe_layer_desc* desc) {
  if (check_desc(desc) != QE_OK) return 0;
  return geom_of(desc).bytes;
}

size_t qe_linear_workspace_bytes(const qe_layer_desc* desc, int32_t T) {
  if (check_desc(desc) != QE_OK || T < 0) return 0;
  // sized for the larger of the fp32 / bf16 input plans
  return std::max(make_plan(desc, T, true).bytes, make_plan(desc, T, false).bytes);
}

qe_status qe_quantize_weights(const qe_layer_desc* desc, const void* W, qe_dtype w_dtype, const float* s,
                              void* w_packed, float* w_scale, float* w_mean, float* w_colmax, float* s_inv,
                              void* stream) {
  qe_status st = check_desc(desc);
  if (st != QE_OK) return st;
  if (!W || !s || !w_packed || !w_scale) return QE_ERR_INVALID_ARG;
  if (w_dtype != QE_F32 && w_dtype != QE_BF16) return QE_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(s) || !aligned16(w_packed) || !aligned16(w_scale) ||
      (w_mean && !aligned16(w_mean)) || (w_colmax && !aligned16(w_colmax)) || (s_inv && !aligned16(s_inv)))
    return QE_ERR_ALIGNMENT;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  QE_CUDA(launch_quantize_weights(W, w_dtype == QE_BF16, s, desc->d_out, desc->d_in, desc->group, desc->w_bits,
                                  static_cast<uint8_t*>(w_packed), w_scale, desc->w_scale_fp16,
                                  device_error_ptr(), cs),
          "quantize_weights");
  if (w_mean || w_colmax)
    QE_CUDA(launch_colstats(W, w_dtype == QE_BF16, desc->d_out, desc->d_in, w_mean, w_colmax, cs), "colstats");
  if (s_inv) QE_CUDA(launch_recip(s, desc->d_in, s_inv, cs), "recip");
  return QE_OK;
}

qe_status qe_pack_adapters(const qe_layer_desc* desc, const void* A_s, const void* B_s, const void* A_r,
                           const void* B_r, const void* G, void* out, void* stream) {
  if (desc && desc->routed_channels != 0) return QE_ERR_INVALID_ARG;  // cluster-sparse: qe_pack_adapters_sparse
  return qe_pack_adapters_sparse(desc, A_s, B_s, nullptr, A_r, B_r, G, out, stream);
}

qe_status qe_pack_adapters_sparse(const qe_layer_desc* desc, const void* A_s, const void* B_s,
                                  const int32_t* channels, const void* A_r, const void* B_r, const void* G, void* out,
                                  void* stream) {
  qe_status st = check_desc(desc);
  if (st != QE_OK) return st;
  if (!G || !out) return QE_ERR_INVALID_ARG;
  if (desc->routed_channels > 0 && !channels) return QE_ERR_INVALID_ARG;
  if (desc->rank_shared > 0 && (!A_s || !B_s)) return QE_ERR_INVALID_ARG;
  if (desc->rank_routed > 0 && (!A_r || !B_r)) return QE_ERR_INVALID_ARG;
  if (!aligned16(out)) return QE_ERR_ALIGNMENT;
  const AdapterGeom g = geom_of(desc);
  QE_CUDA(launch_pack_adapters(g, desc->d_in, desc->d_out, static_cast<const uint16_t*>(A_s),
                               static_cast<const uint16_t*>(B_s), static_cast<const uint16_t*>(A_r),
                               static_cast<const uint16_t*>(B_r), static_cast<const uint16_t*>(G), channels,
                               static_cast<uint8_t*>(out), device_error_ptr(), static_cast<cudaStream_t>(stream)),
          "pack_adapters");
  return QE_OK;
}

qe_status qe_topk_importance(const void* X, qe_dtype x_dtype, const float* w_mean, int32_t T, int32_t d_in,
                             int32_t k, int32_t* idx, int32_t* hist, int32_t accumulate_hist, void* stream) {
  if (T < 0 || d_in <= 0 || k < 1 || k > 128 || k > d_in) return QE_ERR_INVALID_ARG;
  if (d_in % 8 != 0 || d_in > 32768) return QE_ERR_UNSUPPORTED;
  if (x_dtype != QE_F32 && x_dtype != QE_BF16) return QE_ERR_INVALID_ARG;
  if (!w_mean || (T > 0 && (!X || !idx))) return QE_ERR_INVALID_ARG;
  if ((X && !aligned16(X)) || !aligned16(w_mean)) return QE_ERR_ALIGNMENT;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (hist && !accumulate_hist) QE_CUDA(cudaMemsetAsync(hist, 0, size_t(d_in) * 4, cs), "memset hist");
  QE_CUDA(launch_topk(X, x_dtype == QE_BF16, w_mean, T, d_in, k, idx, hist, device_error_ptr(), cs), "topk");
  return QE_OK;
}

qe_status qe_route(const void* X, qe_dtype x_dtype, const void* G, int32_t T, int32_t d_in, int32_t n_routed,
                   int32_t* expert, int32_t* perm, int32_t* offsets, float* logits, void* stream) {
  if (T < 0 || T > (1 << 20) || d_in <= 0 || n_routed < 1 || n_routed > kMaxRouted) return QE_ERR_INVALID_ARG;
  if (d_in % 8 != 0) return QE_ERR_UNSUPPORTED;
  if (x_dtype != QE_F32 && x_dtype != QE_BF16) return QE_ERR_INVALID_ARG;
  if (!G || !expert || !perm || !offsets || (T > 0 && !X)) return QE_ERR_INVALID_ARG;
  if ((X && !aligned16(X)) || !aligned16(G)) return QE_ERR_ALIGNMENT;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // routing alone: no activation scale is computed, so s_inv is not read
  QE_CUDA(launch_route_stats(X, x_dtype == QE_BF16, nullptr, static_cast<const uint16_t*>(G),
                             T, d_in, n_routed, 1, expert, nullptr, logits, cs),
          "route_stats");
  QE_CUDA(launch_bucket(expert, T, n_routed, perm, nullptr, offsets, cs), "bucket");
  return QE_OK;
}

qe_status qe_linear_forward(const qe_layer_desc* desc, const qe_layer_weights* weights, const void* X,
                            qe_dtype x_dtype, int32_t T, void* Y, qe_dtype y_dtype, void* workspace,
                            size_t workspace_bytes, void* stream) {
  return forward_impl(desc, weights, X, x_dtype, T, Y, y_dtype, workspace, workspace_bytes, nullptr, nullptr,
                      nullptr, nullptr, QE_STAGE_ALL, static_cast<cudaStream_t>(stream));
}

int32_t qe_linear_kernel_launches(const qe_layer_desc* desc, int32_t T, qe_dtype x_dtype) {
  if (check_desc(desc) != QE_OK || T < 0) return -1;
  if (T == 0) return 0;
  const Plan p = make_plan(desc, T, x_dtype == QE_BF16);
  int n = (x_dtype == QE_BF16) ? 1 : 3;  // down-projection GEMM (fp32 inputs: split + hi and lo passes)
  n += 1;                                // routing + bucket sort + quantization (cooperative)
  n += 1;                                // main product (int8 GEMM or weight-only)
  if (p.msplits > 1) n += 1;             // split-K reduce
  return n;
}

qe_status qe_linear_plan(const qe_layer_desc* desc, int32_t T, qe_dtype x_dtype, qe_linear_plan_info* out) {
  const qe_status st = check_desc(desc);
  if (st != QE_OK) return st;
  if (!out || T < 1) return QE_ERR_INVALID_ARG;
  if (x_dtype != QE_F32 && x_dtype != QE_BF16) return QE_ERR_INVALID_ARG;
  const Plan p = make_plan(desc, T, x_dtype == QE_BF16);
  out->product_tile_tokens = p.bn;
  out->product_k_splits = p.msplits;
  out->adapter_atoms = p.has_ad ? p.g.R_pad / kAdapterAtom : 0;
  out->adapter_gemm_width = p.g.R_tot;
  out->adapter_gemm_tile = p.up.nu;
  out->adapter_gemm_splits = p.uslots;
  out->weight_only = desc->a_bits == 16 ? 1 : 0;
  out->workspace_bytes = static_cast<int64_t>(p.bytes);
  out->decode_product = p.dec ? 1 : 0;
  out->decode_ctas = p.dec ? p.dp.grid : 0;
  out->decode_max_segments = p.dec ? p.dp.maxseg : 0;
  return QE_OK;
}

qe_status qe_linear_forward_stages(const qe_layer_desc* desc, const qe_layer_weights* weights, const void* X,
                                   qe_dtype x_dtype, int32_t T, void* Y, qe_dtype y_dtype, void* workspace,
                                   size_t workspace_bytes, int32_t stages, void* stream) {
  if (stages & ~QE_STAGE_ALL) return QE_ERR_INVALID_ARG;
  return forward_impl(desc, weights, X, x_dtype, T, Y, y_dtype, workspace, workspace_bytes, nullptr, nullptr,
                      nullptr, nullptr, stages, static_cast<cudaStream_t>(stream));
}

qe_status qe_linear_forward_debug(const qe_layer_desc* desc, const qe_layer_weights* weights, const void* X,
                                  qe_dtype x_dtype, int32_t T, void* Y, qe_dtype y_dtype, void* workspace,
                                  size_t workspace_bytes, int32_t* acc, int32_t* expert, int32_t* perm, float* sa,
                                  void* stream) {
  if (desc && desc->a_bits == 16 && acc) return QE_ERR_UNSUPPORTED;
  return forward_impl(desc, weights, X, x_dtype, T, Y, y_dtype, workspace, workspace_bytes, acc, expert, perm, sa,
                      QE_STAGE_ALL, static_cast<cudaStream_t>(stream));
}

qe_status qe_unpack_weights(const qe_layer_desc* desc, const void* w_packed, int8_t* codes, void* stream) {
  qe_status st = check_desc(desc);
  if (st != QE_OK) return st;
  if (!w_packed || !codes) return QE_ERR_INVALID_ARG;
  QE_CUDA(launch_unpack_weights(static_cast<const uint8_t*>(w_packed), desc->d_out, desc->d_in, desc->w_bits, codes,
                                static_cast<cudaStream_t>(stream)),
          "unpack_weights");
  return QE_OK;
}

qe_status qe_act_quant(const void* X, qe_dtype x_dtype, const float* s_inv, int32_t T, int32_t d_in, int32_t a_bits,
                       int8_t* codes, float* sa, void* stream) {
  if (T < 0 || d_in <= 0 || (a_bits != 6 && a_bits != 8)) return QE_ERR_INVALID_ARG;
  if (d_in % 8 != 0) return QE_ERR_UNSUPPORTED;
  if (x_dtype != QE_F32 && x_dtype != QE_BF16) return QE_ERR_INVALID_ARG;
  if (!s_inv || !sa || (T > 0 && (!X || !codes))) return QE_ERR_INVALID_ARG;
  if ((X && !aligned16(X)) || !aligned16(s_inv) || (codes && (reinterpret_cast<uintptr_t>(codes) & 7u)))
    return QE_ERR_ALIGNMENT;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int qmax = qmax_of(a_bits);
  QE_CUDA(launch_route_stats(X, x_dtype == QE_BF16, s_inv, nullptr, T, d_in, 0, qmax, nullptr, sa, nullptr, cs),
          "act_stats");
  QE_CUDA(launch_act_quant(X, x_dtype == QE_BF16, s_inv, T, d_in, qmax, sa, nullptr, codes, nullptr, nullptr,
                           nullptr, nullptr, cs),
          "act_quant");
  return QE_OK;
}

qe_status qe_linear_forward_noalloc(const qe_layer_desc* desc, const qe_layer_weights* weights, const void* X,
                                    qe_dtype x_dtype, int32_t T, void* Y, qe_dtype y_dtype, void* stream) {
  // the same argument checks as qe_linear_forward, before the scratch is sized
  qe_status s = check_forward_args(desc, weights, X, x_dtype, T, Y, y_dtype);
  if (s != QE_OK || T == 0) return s;
  const size_t need = make_plan(desc, T, x_dtype == QE_BF16).bytes;  // the scratch this input dtype needs
  if (need > QE_NOALLOC_WORKSPACE_BYTES) {
    snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
             "qe_linear_forward_noalloc: this layer needs %zu bytes of scratch for T=%d, above the fixed %u",
             need, T, static_cast<unsigned>(QE_NOALLOC_WORKSPACE_BYTES));
    return QE_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if ((s = static_scratch(&scratch)) != QE_OK) return s;
  return forward_impl(desc, weights, X, x_dtype, T, Y, y_dtype, scratch, QE_NOALLOC_WORKSPACE_BYTES, nullptr,
                      nullptr, nullptr, nullptr, QE_STAGE_ALL, static_cast<cudaStream_t>(stream));
}

const char* qe_status_string(qe_status s) {
  switch (s) {
    case QE_OK: return "ok";
    case QE_ERR_INVALID_ARG: return "invalid argument";
    case QE_ERR_UNSUPPORTED: return "unsupported configuration";
    case QE_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case QE_ERR_WORKSPACE: return "workspace missing or too small";
    case QE_ERR_CUDA: return "CUDA error";
    case QE_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* qe_last_cuda_error(void) { return g_last_cuda_error; }

qe_status qe_device_error(void* stream, int32_t* code, int32_t clear) {
  int v = 0;
  QE_CUDA(read_device_error(&v, clear != 0, static_cast<cudaStream_t>(stream)), "device_error");
  if (code) *code = v;
  return v ? QE_ERR_TIMEOUT : QE_OK;
}

qe_status qe_split_channels(const int32_t* hist, int32_t d_in, int32_t k, int32_t C, int32_t* channel_pos,
                            void* stream) {
  if (d_in < 1 || d_in > (1 << 24) || k < 0 || k > 128 || C < 1 || C > 4096) return QE_ERR_INVALID_ARG;
  if (!hist || !channel_pos) return QE_ERR_INVALID_ARG;
  QE_CUDA(launch_split_channels(hist, d_in, k, C, channel_pos, static_cast<cudaStream_t>(stream)), "split_channels");
  return QE_OK;
}

qe_status qe_cooccurrence_npmi(const int32_t* idx, int32_t T, int32_t k, const int32_t* channel_pos, int32_t d_in,
                               int32_t C, int32_t* O, float* S, float threshold, void* stream) {
  if (T < 0 || T > (1 << 20) || k < 1 || k > 128 || C < 1 || C > 4096 || d_in < 1) return QE_ERR_INVALID_ARG;
  if (!O || !channel_pos || (T > 0 && !idx)) return QE_ERR_INVALID_ARG;
  if (!aligned16(O) || (S && !aligned16(S))) return QE_ERR_ALIGNMENT;
  QE_CUDA(launch_cooc_npmi(idx, T, k, channel_pos, d_in, C, O, S, threshold, static_cast<cudaStream_t>(stream)),
          "cooc_npmi");
  return QE_OK;
}

qe_status qe_selftest_wait_timeout(int32_t limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return QE_ERR_INVALID_ARG;
  int* err = device_error_ptr();
  if (!err) return cuda_fail(cudaErrorInvalidSymbol, "device error word");
  QE_CUDA(launch_wait_selftest(err, static_cast<uint64_t>(limit_us) * 1000ull, static_cast<cudaStream_t>(stream)),
          "wait_selftest");
  return QE_OK;
}

}  // extern "C"
