// C ABI of the MXFP4 MoE expert block: argument checks, workspace carving and the launch
// sequence of the forward and input-gradient backward.  See include/mxfp4_moe.h.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/mxfp4_moe.h"
#include "kernels.h"
#include "aux_kernels.h"

namespace {

constexpr size_t kAlign = 256;
size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct WsLayout {
  size_t err, off, idx, w, perm, inv, w_row, blk_hist, sfb, dgu, act, dh, rows, total;
};

// Row stride of the activation scales the block-scaled gate_up GEMM reads: one byte per
// 32 elements of H, padded to whole k-steps (two blocks each) and to 32 bytes (bulk copies
// want 16; the bank swizzle of the scale words exchanges words within 32-byte groups).
int sfb_stride(int H) { return (2 * ((H + moe::kBK - 1) / moe::kBK) + 31) / 32 * 32; }

// Workspace regions, each 256-byte aligned, in this order.  The forward leaves the routing
// (idx, w, perm, inv, w_row), the GLU derivative factors (dgu) and the expert outputs y in
// expert-sorted row order (rows) for the backward.
WsLayout ws_layout(const mxfp4_moe_dims& d) {
  const size_t A = (size_t)d.T * d.k;
  WsLayout L{};
  size_t o = 0;
  L.err = o;      o = up(o + 16);
  L.off = o;      o = up(o + 4ull * (d.E + 1));
  L.idx = o;      o = up(o + 4 * A);                 // expert of each slot t*k+j
  L.w = o;        o = up(o + 4 * A);                 // routing weight of each slot
  L.perm = o;     o = up(o + 4 * A);                 // sorted row -> slot
  L.inv = o;      o = up(o + 4 * A);                 // slot -> sorted row
  L.w_row = o;    o = up(o + 4 * A);                 // routing weight of each sorted row
  L.blk_hist = o; o = up(o + 4 * moe::route_scratch_words(d.T, d.E));  // routing scratch
  L.sfb = o;      o = up(o + A * sfb_stride(d.H));     // activation scales (gate_up)
  L.dgu = o;      o = up(o + 4 * A * d.I);           // saved GLU derivative factors (bf16 pairs)
  L.act = o;      o = up(o + 2 * A * d.I);           // act [A][I] (the down GEMM's input)
  // dH [A][2I] (backward); in the forward, the E4M3 hi | lo parts of Xp ([A][H] bytes each)
  L.dh = o;       o = up(o + 2 * A * (2 * d.I > d.H ? 2 * d.I : d.H));
  L.rows = o;     o = up(o + 2 * A * d.H);           // y (fwd), dYp -> dX rows (bwd)
  L.total = o;
  return L;
}

struct WtLayout {
  size_t dn_blocks, gu_blocks, dn_scales, gu_scales, total;
};

WtLayout wt_layout(const mxfp4_moe_dims& d) {
  WtLayout L{};
  const size_t E = d.E, H = d.H, I = d.I;
  size_t o = 0;
  L.dn_blocks = o; o = up(o + E * I * (H / 2));
  L.gu_blocks = o; o = up(o + E * H * I);
  L.dn_scales = o; o = up(o + E * (I / 32) * H);
  L.gu_scales = o; o = up(o + E * (H / 32) * 2 * I);
  L.total = o;
  return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(const mxfp4_moe_dims* d) {
  if (!d) return MXFP4_MOE_ERR_INVALID_ARG;
  if (d->T < 1 || d->H < 32 || d->I < 32 || d->H % 32 || d->I % 32) return MXFP4_MOE_ERR_INVALID_ARG;
  if (d->E < 1 || d->E > 256 || d->k < 1 || d->k > d->E) return MXFP4_MOE_ERR_INVALID_ARG;
  if ((long long)d->T * d->k >= (1ll << 31)) return MXFP4_MOE_ERR_INVALID_ARG;
  if (!(d->glu_limit > 0.f) || !(d->glu_alpha == d->glu_alpha)) return MXFP4_MOE_ERR_INVALID_ARG;
  if (d->gate_up_format != MXFP4_MOE_GATE_UP_BF16 &&
      d->gate_up_format != MXFP4_MOE_GATE_UP_BLOCK_SCALED)
    return MXFP4_MOE_ERR_INVALID_ARG;
  // the grouped GEMM keeps a tile's scales for the whole contraction in shared memory
  if (moe::grouped_gemm_smem_bytes(d->H > 2 * d->I ? d->H : 2 * d->I, 0) > 232448 ||
      moe::grouped_gemm_smem_bytes(d->H, sfb_stride(d->H)) > 232448)
    return MXFP4_MOE_ERR_INVALID_ARG;
  return MXFP4_MOE_OK;
}

int check_weights(const mxfp4_moe_weights* w) {
  if (!w || !w->gu_blocks || !w->gu_scales || !w->gu_bias || !w->dn_blocks || !w->dn_scales ||
      !w->dn_bias)
    return MXFP4_MOE_ERR_INVALID_ARG;
  if (!aligned16(w->gu_blocks) || !aligned16(w->gu_scales) || !aligned16(w->dn_blocks) ||
      !aligned16(w->dn_scales) || !aligned16(w->gu_bias) || !aligned16(w->dn_bias))
    return MXFP4_MOE_ERR_INVALID_ARG;
  return MXFP4_MOE_OK;
}

// Current device must be sm_100 (B200).  Returns the SM count through `sms`.
int check_device(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MXFP4_MOE_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return MXFP4_MOE_ERR_CUDA;
  if (major != 10 || minor != 0) return MXFP4_MOE_ERR_UNSUPPORTED_DEVICE;
  if (sms && cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MXFP4_MOE_ERR_CUDA;
  return MXFP4_MOE_OK;
}

// Largest fp32 x such that bf16(x) <= limit under round-to-nearest-even: the clamp-mask
// decision "bf16(h) <= limit" becomes one fp32 compare.  For limit = 7 this is 7.015625
// (the tie between 7 and the next bf16, 7.03125, rounds to 7, whose mantissa is even).
float bf16_mask_limit(float limit) {
  uint32_t b;
  std::memcpy(&b, &limit, 4);
  // largest bf16 value <= limit (truncate the fp32 pattern toward zero for positive limits)
  uint32_t lo = b & 0xFFFF0000u;
  float flo;
  std::memcpy(&flo, &lo, 4);
  const uint32_t hi = lo + 0x10000u;  // next bf16 up
  float fhi;
  std::memcpy(&fhi, &hi, 4);
  const double mid = 0.5 * ((double)flo + (double)fhi);  // exact in fp32 (one extra bit)
  float m = (float)mid;
  const bool lo_even = ((lo >> 16) & 1u) == 0;
  if (!lo_even) m = std::nextafter(m, 0.0f);  // a tie would round up to the odd neighbour... of hi
  return m;
}

#define MOE_TRY(expr)                                  \
  do {                                                 \
    cudaError_t e_ = (expr);                           \
    if (e_ != cudaSuccess) return MXFP4_MOE_ERR_CUDA;  \
  } while (0)

template <class T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
}

// ---- per-kernel event timing (mxfp4_moe_profile_begin / _end) -------------------------
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
};
struct Profiler {
  bool on = false;
  std::vector<ProfRec> recs;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
};
Profiler& prof() {
  static Profiler p;
  return p;
}

// Brackets one kernel launch with an event pair when profiling is on.
struct Timed {
  const char* name;
  cudaStream_t st;
  cudaEvent_t a = nullptr;
  Timed(const char* n, cudaStream_t s) : name(n), st(s) {
    nvtxRangePushA(n);  // one NVTX range per kernel launch (free when no tool is attached)
    if (prof().on) {
      a = prof().get();
      cudaEventRecord(a, st);
    }
  }
  ~Timed() {
    nvtxRangePop();
    if (a) {
      cudaEvent_t b = prof().get();
      cudaEventRecord(b, st);
      prof().recs.push_back({name, a, b});
    }
  }
};

#define MOE_LAUNCH(name, expr)   \
  do {                           \
    Timed timed_(name, st);      \
    MOE_TRY(expr);               \
  } while (0)

}  // namespace

extern "C" {

int mxfp4_moe_workspace_size(const mxfp4_moe_dims* d, size_t* bytes) {
  const int rc = check_dims(d);
  if (rc) return rc;
  if (!bytes) return MXFP4_MOE_ERR_INVALID_ARG;
  *bytes = ws_layout(*d).total;
  return MXFP4_MOE_OK;
}

int mxfp4_moe_transposed_weights_size(const mxfp4_moe_dims* d, size_t* bytes) {
  const int rc = check_dims(d);
  if (rc) return rc;
  if (!bytes) return MXFP4_MOE_ERR_INVALID_ARG;
  *bytes = wt_layout(*d).total;
  return MXFP4_MOE_OK;
}

int mxfp4_moe_transpose_weights(const mxfp4_moe_dims* d, const mxfp4_moe_weights* w, void* wt,
                                size_t wt_bytes, void* stream) {
  int rc = check_dims(d);
  if (!rc) rc = check_weights(w);
  if (rc) return rc;
  if (!wt || !aligned16(wt)) return MXFP4_MOE_ERR_INVALID_ARG;
  const WtLayout L = wt_layout(*d);
  if (wt_bytes < L.total) return MXFP4_MOE_ERR_WORKSPACE_TOO_SMALL;
  rc = check_device(nullptr);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_LAUNCH("transpose_packed", moe::launch_transpose_packed(w->dn_blocks, d->E, d->H, d->I, at<uint8_t>(wt, L.dn_blocks), st));
  MOE_LAUNCH("transpose_packed", moe::launch_transpose_packed(w->gu_blocks, d->E, 2 * d->I, d->H, at<uint8_t>(wt, L.gu_blocks), st));
  MOE_LAUNCH("transpose_scales", moe::launch_transpose_scales(w->dn_scales, d->E, d->H, d->I, at<uint8_t>(wt, L.dn_scales), st));
  MOE_LAUNCH("transpose_scales", moe::launch_transpose_scales(w->gu_scales, d->E, 2 * d->I, d->H, at<uint8_t>(wt, L.gu_scales), st));
  return MXFP4_MOE_OK;
}

int mxfp4_moe_forward(const mxfp4_moe_dims* d, const mxfp4_moe_weights* w, const uint16_t* x,
                      const float* logits, uint16_t* y, int32_t* topk_idx, float* topk_w,
                      void* ws, size_t ws_bytes, void* stream) {
  int rc = check_dims(d);
  if (!rc) rc = check_weights(w);
  if (rc) return rc;
  if (!x || !logits || !y || !ws || !aligned16(x) || !aligned16(y) || !aligned16(ws) ||
      (reinterpret_cast<uintptr_t>(logits) & 3u))
    return MXFP4_MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*d);
  if (ws_bytes < L.total) return MXFP4_MOE_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  rc = check_device(&sms);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int T = d->T, H = d->H, I = d->I, E = d->E, k = d->k, A = T * k;
  int* err = at<int>(ws, L.err);
  int32_t* off = at<int32_t>(ws, L.off);
  int32_t* idx = at<int32_t>(ws, L.idx);
  float* wr = at<float>(ws, L.w);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* inv = at<int32_t>(ws, L.inv);
  float* w_row = at<float>(ws, L.w_row);
  int32_t* blk_hist = at<int32_t>(ws, L.blk_hist);
  uint16_t* dgu = at<uint16_t>(ws, L.dgu);
  uint16_t* act = at<uint16_t>(ws, L.act);
  uint16_t* rows = at<uint16_t>(ws, L.rows);

  MOE_LAUNCH("router_topk", moe::launch_router_topk(logits, T, E, k, idx, wr, blk_hist, topk_idx, topk_w, st));
  MOE_LAUNCH("seg_scan", moe::launch_seg_scan(T, E, blk_hist, st));
  MOE_LAUNCH("build_perm", moe::launch_build_perm(idx, wr, T, E, k, blk_hist, off, perm, inv, w_row, err, st));
  const bool bs = d->gate_up_format == MXFP4_MOE_GATE_UP_BLOCK_SCALED;
  // Xp in expert-sorted order: bf16 rows (in `rows`, which the down GEMM overwrites with y), or
  // as two E4M3 parts (hi | lo in the dH region, free until the backward) with UE8M0 scales
  uint8_t* xhi = at<uint8_t>(ws, L.dh);
  uint8_t* xlo = xhi + (size_t)A * H;
  uint8_t* sfb = at<uint8_t>(ws, L.sfb);
  if (bs)
    MOE_LAUNCH("gather_x_mx", moe::launch_gather_quant(x, H, k, perm, A, xhi, xlo, sfb, sfb_stride(H), err, st));
  else
    MOE_LAUNCH("gather_x", moe::launch_gather_rows(x, H, k, perm, A, rows, nullptr, err, st));

  moe::GemmArgs g{};
  g.off = off; g.E = E; g.A = A; g.err = err;
  g.alpha = d->glu_alpha; g.limit = d->glu_limit; g.mask_limit = bf16_mask_limit(d->glu_limit);
  // gate_up: h = Xp W_gu^T + b_gu; act = GLU(h) and the GLU derivative factors are saved
  // (block-scaled: E2M1 weights against the E4M3 parts; both forms accumulate in fp32)
  g.scales = w->gu_scales; g.K = H; g.N = 2 * I; g.bias = w->gu_bias; g.out0 = dgu; g.out1 = act;
  if (bs) {
    g.tok_lo = xlo; g.sfb = sfb; g.sfb_stride = sfb_stride(H);
    MOE_LAUNCH("gemm_gate_up_glu", moe::launch_grouped_gemm(moe::kEpiGateUp, false, xhi, w->gu_blocks, g, sms, st));
    g.tok_lo = nullptr; g.sfb = nullptr; g.sfb_stride = 0;
  } else {
    MOE_LAUNCH("gemm_gate_up_glu", moe::launch_grouped_gemm(moe::kEpiGateUp, false, rows, w->gu_blocks, g, sms, st));
  }
  // down: y = act W_d^T + b_d per sorted row (kept for the backward's routing-weight gradient)
  g.scales = w->dn_scales; g.K = I; g.N = H; g.bias = w->dn_bias; g.out0 = rows; g.out1 = nullptr;
  MOE_LAUNCH("gemm_down", moe::launch_grouped_gemm(moe::kEpiDown, false, act, w->dn_blocks, g, sms, st));
  // out_t = sum_j w_{t,j} y_{t,j}
  MOE_LAUNCH("combine_y", moe::launch_combine(rows, inv, wr, T, k, H, y, err, st));
  return MXFP4_MOE_OK;
}

int mxfp4_moe_backward_input(const mxfp4_moe_dims* d, const mxfp4_moe_weights* w,
                             const void* wt, size_t wt_bytes, const uint16_t* dy, void* ws,
                             size_t ws_bytes, uint16_t* dx, float* d_topk_w, float* d_logits,
                             void* stream) {
  int rc = check_dims(d);
  if (!rc) rc = check_weights(w);
  if (rc) return rc;
  if (!wt || !dy || !ws || !dx || !d_topk_w || !aligned16(wt) || !aligned16(dy) ||
      !aligned16(ws) || !aligned16(dx) || !aligned16(d_topk_w) ||
      (d_logits && !aligned16(d_logits)))
    return MXFP4_MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*d);
  const WtLayout LT = wt_layout(*d);
  if (ws_bytes < L.total || wt_bytes < LT.total) return MXFP4_MOE_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  rc = check_device(&sms);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int T = d->T, H = d->H, I = d->I, E = d->E, k = d->k, A = T * k;
  void* wtp = const_cast<void*>(wt);
  int* err = at<int>(ws, L.err);
  int32_t* off = at<int32_t>(ws, L.off);
  int32_t* idx = at<int32_t>(ws, L.idx);
  float* wr = at<float>(ws, L.w);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* inv = at<int32_t>(ws, L.inv);
  const float* w_row = at<float>(ws, L.w_row);
  const uint32_t* dgu = at<uint32_t>(ws, L.dgu);
  uint16_t* dh = at<uint16_t>(ws, L.dh);
  uint16_t* rows = at<uint16_t>(ws, L.rows);

  // d_topk_w[slot] = <dY_t, y_r> with the forward's y_r read in place, then dYp[r] = dY[t(r)]
  MOE_LAUNCH("gather_dy_dw", moe::launch_gather_rows(dy, H, k, perm, A, rows, d_topk_w, err, st));
  moe::GemmArgs g{};
  g.off = off; g.E = E; g.A = A; g.err = err;
  g.alpha = d->glu_alpha; g.limit = d->glu_limit;
  // dZ = dYp W_d (contract over H); epilogue: dact = w dZ, dH = dact * saved GLU factors
  g.scales = at<uint8_t>(wtp, LT.dn_scales); g.K = H; g.N = I; g.out0 = dh; g.dgu = dgu; g.w_row = w_row;
  MOE_LAUNCH("gemm_dact_glu_bwd", moe::launch_grouped_gemm(moe::kEpiDact, true, rows, at<uint8_t>(wtp, LT.dn_blocks), g, sms, st));
  // dx = dH W_gu (contract over the 2I interleaved rows), per sorted row
  g.scales = at<uint8_t>(wtp, LT.gu_scales); g.K = 2 * I; g.N = H; g.out0 = rows; g.dgu = nullptr; g.w_row = nullptr;
  MOE_LAUNCH("gemm_dx", moe::launch_grouped_gemm(moe::kEpiDx, true, dh, at<uint8_t>(wtp, LT.gu_blocks), g, sms, st));
  MOE_LAUNCH("combine_dx", moe::launch_combine(rows, inv, nullptr, T, k, H, dx, err, st));
  MOE_LAUNCH("router_backward", moe::launch_router_backward(idx, wr, d_topk_w, T, E, k, d_logits, st));
  return MXFP4_MOE_OK;
}

int mxfp4_moe_grouped_matmul(int32_t E, int32_t N, int32_t K, int32_t A, const int32_t* off,
                             const uint16_t* x, const uint8_t* blocks, const uint8_t* scales,
                             int32_t transposed, uint16_t* out, int32_t* err_word, void* stream) {
  if (E < 1 || E > 256 || N < 32 || N % 32 || K < 32 || K % 32 || A < 0 || !off || !x ||
      !blocks || !scales || !out || !aligned16(x) || !aligned16(blocks) || !aligned16(scales) ||
      !aligned16(out) || (transposed != 0 && transposed != 1))
    return MXFP4_MOE_ERR_INVALID_ARG;
  if (moe::grouped_gemm_smem_bytes(K, 0) > 232448) return MXFP4_MOE_ERR_INVALID_ARG;
  int sms = 0;
  const int rc = check_device(&sms);
  if (rc) return rc;
  if (A == 0) return MXFP4_MOE_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  moe::GemmArgs g{};
  g.off = off; g.E = E; g.A = A; g.err = reinterpret_cast<int*>(err_word);
  g.scales = scales; g.K = K; g.N = N; g.out0 = out;
  MOE_LAUNCH("grouped_matmul", moe::launch_grouped_gemm(moe::kEpiDx, transposed != 0, x, blocks, g, sms, st));
  return MXFP4_MOE_OK;
}

int mxfp4_moe_dequantize(const uint8_t* blocks, const uint8_t* scales, int64_t rows, int64_t K,
                         uint16_t* out, void* stream) {
  if (!blocks || !scales || !out || rows < 0 || K < 32 || K % 32 || !aligned16(blocks) ||
      !aligned16(out))
    return MXFP4_MOE_ERR_INVALID_ARG;
  const int rc = check_device(nullptr);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_LAUNCH("dequant", moe::launch_dequant(blocks, scales, rows, K, out, st));
  return MXFP4_MOE_OK;
}

int mxfp4_moe_interleave_gate_up(const mxfp4_moe_dims* d, const uint8_t* stacked_blocks,
                                 const uint8_t* stacked_scales, const uint16_t* stacked_bias,
                                 uint8_t* blocks, uint8_t* scales, uint16_t* bias, void* stream) {
  if (!d || !stacked_blocks || !stacked_scales || !stacked_bias || !blocks || !scales || !bias)
    return MXFP4_MOE_ERR_INVALID_ARG;
  if (d->E < 1 || d->E > 256 || d->H < 32 || d->H % 32 || d->I < 32 || d->I % 32)
    return MXFP4_MOE_ERR_INVALID_ARG;
  if (!aligned16(stacked_blocks) || !aligned16(blocks)) return MXFP4_MOE_ERR_INVALID_ARG;
  const int rc = check_device(nullptr);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_LAUNCH("interleave_gate_up",
             moe::launch_interleave_gate_up(stacked_blocks, stacked_scales, stacked_bias, d->E, d->I,
                                            d->H, blocks, scales, bias, st));
  return MXFP4_MOE_OK;
}

int mxfp4_moe_residual_router(int32_t T, int32_t H, int32_t E, const uint16_t* x,
                              const uint16_t* y, const uint16_t* w_r, const uint16_t* b_r,
                              uint16_t* x_out, float* logits, void* stream) {
  if (T < 0 || H < 32 || H % 32 || E < 1 || E > 256 || !x || !aligned16(x))
    return MXFP4_MOE_ERR_INVALID_ARG;
  if (!y && !logits) return MXFP4_MOE_ERR_INVALID_ARG;
  if ((y == nullptr) != (x_out == nullptr)) return MXFP4_MOE_ERR_INVALID_ARG;
  if (y && (!aligned16(y) || !aligned16(x_out))) return MXFP4_MOE_ERR_INVALID_ARG;
  if (logits && (!w_r || !aligned16(w_r))) return MXFP4_MOE_ERR_INVALID_ARG;
  if (x_out) {  // x_out overlapping x or y would be read after being written
    const size_t n = 2 * (size_t)T * H;
    auto overlaps = [n](const void* a, const void* b) {
      const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
      return pa < pb + n && pb < pa + n;
    };
    if (T > 0 && (overlaps(x_out, x) || overlaps(x_out, y))) return MXFP4_MOE_ERR_INVALID_ARG;
  }
  const int rc = check_device(nullptr);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_LAUNCH("residual_router",
             moe::launch_residual_router(T, H, E, x, y, w_r, b_r, x_out, logits, st));
  return MXFP4_MOE_OK;
}

int mxfp4_moe_grad_chain(int32_t T, int32_t H, int32_t E, const uint16_t* g, const uint16_t* dx,
                         const float* d_logits, const uint16_t* w_r, uint16_t* g_out,
                         void* stream) {
  if (T < 0 || H < 32 || H % 32 || E < 1 || E > 256 || !g || !dx || !d_logits || !w_r || !g_out ||
      !aligned16(g) || !aligned16(dx) || !aligned16(w_r) || !aligned16(g_out))
    return MXFP4_MOE_ERR_INVALID_ARG;
  const int rc = check_device(nullptr);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_LAUNCH("grad_chain", moe::launch_grad_chain(T, H, E, g, dx, d_logits, w_r, g_out, st));
  return MXFP4_MOE_OK;
}

int mxfp4_moe_selftest_wait_timeout(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < 16 || !aligned16(ws)) return MXFP4_MOE_ERR_INVALID_ARG;
  const int rc = check_device(nullptr);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_LAUNCH("selftest_wait_timeout", moe::launch_wait_timeout_selftest(static_cast<int*>(ws), st));
  return MXFP4_MOE_OK;
}

int mxfp4_moe_check(void* ws, void* stream, int32_t* where) {
  if (!ws) return MXFP4_MOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MXFP4_MOE_ERR_CUDA;
  int word[2] = {0, 0};
  if (cudaMemcpy(word, ws, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MXFP4_MOE_ERR_CUDA;
  if (word[0] != 0 && cudaMemset(ws, 0, sizeof(word)) != cudaSuccess) return MXFP4_MOE_ERR_CUDA;
  if (where) *where = word[1];
  return word[0];
}

int mxfp4_moe_profile_begin(void) {
  prof().on = true;
  return MXFP4_MOE_OK;
}

int mxfp4_moe_profile_end(mxfp4_moe_kernel_time* out, int32_t max, int32_t* n) {
  if (!out || !n || max < 0) return MXFP4_MOE_ERR_INVALID_ARG;
  Profiler& P = prof();
  P.on = false;
  int rc = MXFP4_MOE_OK;
  int cnt = 0;
  for (const ProfRec& r : P.recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
      rc = MXFP4_MOE_ERR_CUDA;
    int i = 0;
    while (i < cnt && i < max && std::strncmp(out[i].name, r.name, sizeof(out[i].name)) != 0) ++i;
    if (i == cnt && cnt < max) {
      std::memset(&out[i], 0, sizeof(out[i]));
      std::strncpy(out[i].name, r.name, sizeof(out[i].name) - 1);
      ++cnt;
    }
    if (i < cnt) {
      out[i].launches += 1;
      out[i].total_ms += ms;
    }
    P.pool.push_back(r.a);
    P.pool.push_back(r.b);
  }
  P.recs.clear();
  *n = cnt;
  return rc;
}

int mxfp4_moe_build_flags(void) { return MXFP4_MOE_DEBUG ? MXFP4_MOE_BUILD_DEBUG : 0; }

const char* mxfp4_moe_strerror(int code) {
  switch (code) {
    case MXFP4_MOE_OK: return "ok";
    case MXFP4_MOE_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, or unsupported shape)";
    case MXFP4_MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace smaller than the size query returned";
    case MXFP4_MOE_ERR_UNSUPPORTED_DEVICE: return "current CUDA device is not sm_100 (B200)";
    case MXFP4_MOE_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
    case MXFP4_MOE_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait expired";
    case MXFP4_MOE_ERR_DEVICE_BOUNDS: return "a device-side index check failed";
    default: return "unknown error code";
  }
}

}  // extern "C"
