// C ABI of the decode library: argument checks, workspace layout, launches.
// Declarations and argument contracts: include/dejavu.h.
#include <atomic>
#include <cstdlib>
#include <map>
#include <cstring>
#include <mutex>

#include "../../include/dejavu.h"
#include "dv_api_kernels.cuh"
#include "dv_launchers.cuh"
#include "dv_tc_launch.h"

using namespace dv;
using bf16 = __nv_bfloat16;

namespace {


constexpr int ATTN_S_MIN = 32;
// Every layout starts with the same fixed header that holds the counters, so
// calls of different operations may share one workspace: the status word at
// 0, the selection tickets at 16, 32, 48 and 64, and the attention split
// counters [B][kh_max] from 1024.
constexpr size_t WS_HEADER = 72 * 1024;
constexpr int KH_LIMIT = 1000;  // B * kh_max counters must fit the header

// Workspace layout. Offsets in bytes from the workspace base.
struct Layout {
  size_t status, sel_ticket_h, sel_ticket_m, pa_ticket, pb_ticket, attn_ctr, t1;
  size_t yA, yM, z, scores_h, bm_h, head_idx, head_count, scores, bm_m, idx, count;
  size_t q, part, H, seg_idx, seg_a, seg_cnt, tc_x, tc_act, tc_rowid, tc_tiles, tc_red, tc_tick, tc_acc, total;
  int nseg, SEG, nsplit_max, KC, XC;
};

bool dims_ok(const dv_dims& D) {
  return D.B >= 1 && D.B <= 16 && D.d >= 8 && D.d % 8 == 0 && D.N >= 1 && D.r >= 0 && D.r % 8 == 0 &&
         D.h >= 0 && D.dh >= 0 && D.cap >= 0 && D.k_max >= 0 && D.kh_max >= 0 && D.k_max <= D.N &&
         D.kh_max <= (D.h > 0 ? D.h : 0) && D.kh_max <= KH_LIMIT;
}

Layout layout(const dv_dims& D, int wbytes) {
  Layout L = {};
  const int B = D.B;
  const int E = 16 / wbytes;
  L.SEG = GEMV_WARPS * rpw_for(D.d, E);
  L.nseg = (D.k_max + L.SEG - 1) / L.SEG;
  L.nsplit_max = (D.cap + ATTN_S_MIN - 1) / ATTN_S_MIN;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o += up256(bytes); return r; };
  L.status = take(WS_HEADER);
  L.sel_ticket_h = L.status + 16;
  L.sel_ticket_m = L.status + 32;
  L.pa_ticket = L.status + 48;
  L.pb_ticket = L.status + 64;
  L.attn_ctr = L.status + 1024;
  L.t1 = take(4ull * B * D.d);
  L.yA = take(4ull * B * D.d);
  L.yM = take(4ull * B * D.d);
  L.z = take(4ull * B * D.r);
  L.scores_h = take(4ull * B * D.h);
  L.bm_h = take(4ull * B * ((D.h + 31) / 32));
  L.head_idx = take(4ull * (D.h > 0 ? D.h : 1));
  L.head_count = take(4);
  L.scores = take(4ull * B * D.N);
  L.bm_m = take(4ull * B * ((D.N + 31) / 32));
  L.idx = take(4ull * D.N);
  L.count = take(4);
  L.q = take(4ull * B * D.kh_max * D.dh);
  L.part = take(4ull * B * D.kh_max * L.nsplit_max * (D.dh + 2));
  L.H = take(4ull * B * D.kh_max * D.dh);
  L.seg_idx = take(4ull * L.nseg * L.SEG);
  L.seg_a = take(4ull * L.nseg * L.SEG * B);
  L.seg_cnt = take(4ull * (L.nseg > 0 ? L.nseg : 1));
  // tensor-core path: the operand split into bf16 hi / lo rows [16][XC]
  // (LN output or the attention outputs H), and the MLP's activations
  // compacted per tile of 128 selected neurons, hi / lo rows [16][KC]
  const int tiles = tc_tiles(D.k_max);
  L.KC = tiles * TC_M;
  L.XC = D.d > D.kh_max * D.dh ? D.d : D.kh_max * D.dh;
  if (L.XC < D.r) L.XC = D.r;
  L.tc_x = take(2ull * 2 * TC_N * L.XC);
  L.tc_act = take(2ull * 2 * TC_N * (L.KC > 0 ? L.KC : 1));
  L.tc_rowid = take(4ull * (L.KC > 0 ? L.KC : 1));
  L.tc_tiles = take(4ull * (tiles > 0 ? tiles : 1));
  // partial-sum slots ([16][128] each) and tickets of the tensor-core
  // reductions: split K of Q/K/V, W1 and the predictor's dense GEMMs, and the
  // row groups of W2 and W^O
  L.tc_red = take(4ull * tc_red_floats(D.k_max, D.kh_max, D.dh, D.d));
  L.tc_tick = take(4ull * tc_tick_count(D.k_max, D.kh_max, D.dh, D.d));
  // fixed-point accumulator of the W2 and W^O partial sums [16][d]
  L.tc_acc = take(8ull * TC_N * D.d);
  L.total = o;
  return L;
}

template <typename P>
P* at(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<char*>(ws) + off);
}

dv_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DV_OK : DV_ERR_CUDA; }

#define DV_TRY(expr)                          \
  do {                                        \
    cudaError_t _e = (expr);                  \
    if (_e != cudaSuccess) return DV_ERR_CUDA; \
  } while (0)

#define DV_CHECK(expr)            \
  do {                            \
    dv_status _s = (expr);        \
    if (_s != DV_OK) return _s;   \
  } while (0)

// Tensor-core path for batch 5..16 (defined below)
bool tc_ok(int B, int d, dv_dtype wdt, int dh, int k_max);
dv_status tc_mlp(const Layout& L, void* ws, const float* y, int B, int d, int N, const void* W1t, const float* b1,
                 const void* W2t, const float* b2, const int32_t* idx, const int32_t* count, int k_max, float* out,
                 int act, cudaStream_t st);
dv_status tc_qkv(const Layout& L, void* ws, const float* y, int B, int d, int h, int dh, const void* Wqkv,
                 const float* bqkv, void* Kc, void* Vc, int cap, int pos, const int32_t* head_idx,
                 const int32_t* head_count, int kh_max, cudaStream_t st);
dv_status tc_wo(const Layout& L, void* ws, int B, int d, int h, int dh, const void* WOt, const float* bO,
                const int32_t* head_idx, const int32_t* head_count, int kh_max, float* out, cudaStream_t st);

// Selection of B score rows of length n: one thread-block cluster per row
// (select_rows_kernel) up to SR_MAX_N scores per row, the one-CTA-per-row
// select_kernel beyond. DV_SELROWS=0 keeps select_kernel for every n.
bool sel_rows_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("DV_SELROWS");
    return !(e && e[0] == '0');
  }();
  return on;
}

cudaError_t select_any(const float* scores, int nrows, int n, int k, float tau, int mode, uint32_t* bm,
                       unsigned* ticket, int32_t* idx, int32_t* count, cudaStream_t st) {
  if (n <= SR_MAX_N && sel_rows_enabled()) {
    SelectRowsArgs a{scores, n, nrows, k, mode, tau, bm, ticket, idx, count};
    return launch_cluster(select_rows_kernel, dim3(SR_CS, nrows), dim3(SR_THREADS), 0, st, SR_CS, a);
  }
  return run_select(scores, nrows, n, k, tau, mode, bm, ticket, idx, count, st);
}

// ---------------------------------------------------------------------------
// Operation bodies shared by the public entry points
// ---------------------------------------------------------------------------

bool fused_enabled();
bool tc_enabled();
int wbytes_of(dv_dtype t);

// A predictor GEMM at batch >= 3 on the tensor cores (tc_dense_kernel):
// out[b][row] = W[row] . x[b] (+ bias[row]), x [B][K] split into the
// workspace's hi / lo operand rows first.
bool pred_tc_ok(int B, dv_dtype wdt, int nrows, int K) {
  return tc_enabled() && B >= 3 && tc_dense_ok(B, wbytes_of(wdt), nrows, K);
}

cudaError_t pred_tc(const Layout& L, void* ws, const void* W, int nrows, int K, const float* bias, const float* x, int B,
                    float* out, long long ldo, cudaStream_t st, bool split = true) {
  bf16* xhi = at<bf16>(ws, L.tc_x);
  bf16* xlo = xhi + (size_t)TC_N * L.XC;
  if (split) {  // (not when the previous call split the same x)
    cudaError_t e = run_tc_split(x, B, K, K, xhi, xlo, K, st);
    if (e != cudaSuccess) return e;
  }
  return run_tc_dense(nullptr, 0, nullptr, nullptr, 0, static_cast<const bf16*>(W), nrows, bias, out, ldo, K, xhi, xlo,
                      B, at<float>(ws, L.tc_red), at<unsigned>(ws, L.tc_tick), at<int>(ws, L.status), st);
}

// The predictor's two stages: z = y A (predict_a_kernel family; rows of At
// read once for all batch rows) and the neuron scores z B^T + b1
// (predict_b_kernel); at batch >= 3 both on the tensor cores. DV_FUSED=0
// runs them as plain GEMVs instead.
cudaError_t predict_z(const Layout& L, void* ws, const float* y, int B, int d, int r, const void* At, dv_dtype dt,
                      float* z, cudaStream_t st) {
  if (!fused_enabled()) return run_gemv(dt, At, r, d, y, d, B, nullptr, z, r, st);
  if (pred_tc_ok(B, dt, r, d)) return pred_tc(L, ws, At, r, d, nullptr, y, B, z, r, st);
  PredictAArgs a = {};
  a.y = y;
  a.At = At;
  a.r = r;
  a.d = d;
  a.nb = B;
  a.z = z;
  return run_predict_a_any_dt(dt, a, st);
}

cudaError_t predict_scores(const Layout& L, void* ws, const float* z, int B, int r, int N, const void* Bm,
                           const float* b1, dv_dtype dt, float* scores, cudaStream_t st) {
  if (!fused_enabled()) return run_gemv(dt, Bm, N, r, z, r, B, b1, scores, N, st);
  if (pred_tc_ok(B, dt, N, r)) return pred_tc(L, ws, Bm, N, r, b1, z, B, scores, N, st);
  PredictBArgs b = {};
  b.z = z;
  b.Bm = Bm;
  b.b1 = b1;
  b.N = N;
  b.r = r;
  b.nb = B;
  b.scores = scores;
  return run_predict_b_dt(dt, b, st);
}

dv_status do_predict_mlp(const Layout& L, void* ws, const float* y, int B, int d, int r, int N, const void* At,
                         const void* Bm, const float* b1, dv_dtype dt, int k, float tau, int mode, float* scores,
                         int32_t* idx, int32_t* count, cudaStream_t st) {
  float* z = at<float>(ws, L.z);
  DV_TRY(predict_z(L, ws, y, B, d, r, At, dt, z, st));
  DV_TRY(predict_scores(L, ws, z, B, r, N, Bm, b1, dt, scores, st));
  DV_TRY(select_any(scores, B, N, k, tau, mode, at<uint32_t>(ws, L.bm_m), at<unsigned>(ws, L.sel_ticket_m), idx, count,
                    st));
  return DV_OK;
}

dv_status do_predict_heads(const Layout& L, void* ws, const float* y, int B, int d, int h, const void* PA, dv_dtype dt,
                           int k_h, float tau, int mode, float* scores, int32_t* head_idx, int32_t* head_count,
                           cudaStream_t st) {
  if (fused_enabled() && pred_tc_ok(B, dt, h, d)) {
    DV_TRY(pred_tc(L, ws, PA, h, d, nullptr, y, B, scores, h, st));
  } else if (fused_enabled()) {
    PredictAArgs a = {};
    a.y = y;
    a.PA = PA;
    a.h = h;
    a.d = d;
    a.nb = B;
    a.scores_h = scores;
    DV_TRY(run_predict_a_any_dt(dt, a, st));
  } else {
    DV_TRY(run_gemv(dt, PA, h, d, y, d, B, nullptr, scores, h, st));
  }
  DV_TRY(select_any(scores, B, h, k_h, tau, mode, at<uint32_t>(ws, L.bm_h), at<unsigned>(ws, L.sel_ticket_h), head_idx,
                    head_count, st));
  return DV_OK;
}

dv_status do_sparse_mlp(const Layout& L, void* ws, const float* y, int B, int d, int N, const void* W1t,
                        const float* b1, const void* W2t, const float* b2, dv_dtype dt, const int32_t* idx,
                        const int32_t* count, int k_max, float* out, int accumulate, int act, cudaStream_t st) {
  if (!accumulate) DV_TRY(cudaMemsetAsync(out, 0, 4ull * B * d, st));
  if (tc_ok(B, d, dt, 64, k_max)) return tc_mlp(L, ws, y, B, d, N, W1t, b1, W2t, b2, idx, count, k_max, out, act, st);
  int* status = at<int>(ws, L.status);
  int32_t* seg_idx = at<int32_t>(ws, L.seg_idx);
  float* seg_a = at<float>(ws, L.seg_a);
  int32_t* seg_cnt = at<int32_t>(ws, L.seg_cnt);
  if (L.nseg == 0) {
    if (b2) {  // nothing selected: out (+)= b2 only
      RowsHeads none{idx, count, nullptr, 0, 1, 0};
      return cuda_status(run_axpy_dt(dt, W2t, d, N, none, b2, out, B, 1, 0, status, st));
    }
    return DV_OK;
  }
  DV_TRY(run_mlp_up_dt(dt, W1t, d, N, y, B, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, L.nseg, act, st));
  RowsMlp src{seg_idx, seg_a, seg_cnt, L.nseg, L.SEG};
  const size_t smem = 4ull * (L.nseg + 1);
  return cuda_status(run_axpy_dt(dt, W2t, d, N, src, b2, out, B, k_max, smem, status, st));
}

dv_status do_sparse_mha(const Layout& L, void* ws, const float* y, int B, int d, int h, int dh, const void* Wqkv,
                        const float* bqkv, const void* WOt, const float* bO, dv_dtype dt, void* Kc, void* Vc, int cap,
                        int pos, float scale, const int32_t* head_idx, const int32_t* head_count, int kh_max,
                        float* out, int accumulate, cudaStream_t st) {
  if (!accumulate) DV_TRY(cudaMemsetAsync(out, 0, 4ull * B * d, st));
  int* status = at<int>(ws, L.status);
  if (tc_ok(B, d, dt, dh, 0)) {
    if (kh_max > 0) {
      DV_CHECK(tc_qkv(L, ws, y, B, d, h, dh, Wqkv, bqkv, Kc, Vc, cap, pos, head_idx, head_count, kh_max, st));
      DV_TRY(run_attn_dt(dt, dh, at<float>(ws, L.q), Kc, Vc, B, h, cap, pos, scale, head_idx, head_count, kh_max,
                         at<float>(ws, L.part), at<unsigned>(ws, L.attn_ctr), at<float>(ws, L.H), status, st));
    }
    return tc_wo(L, ws, B, d, h, dh, WOt, bO, head_idx, head_count, kh_max, out, st);
  }
  if (kh_max == 0) {
    if (bO) {
      RowsHeads none{head_idx, head_count, nullptr, 0, dh, h};
      return cuda_status(run_axpy_dt(dt, WOt, d, h * dh, none, bO, out, B, 1, 0, status, st));
    }
    return DV_OK;
  }
  float* q = at<float>(ws, L.q);
  float* H = at<float>(ws, L.H);
  DV_TRY(run_qkv_dt(dt, Wqkv, d, h, dh, y, B, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos, status, st));
  DV_TRY(run_attn_dt(dt, dh, q, Kc, Vc, B, h, cap, pos, scale, head_idx, head_count, kh_max, at<float>(ws, L.part),
                     at<unsigned>(ws, L.attn_ctr), H, status, st));
  RowsHeads src{head_idx, head_count, H, kh_max, dh, h};
  return cuda_status(run_axpy_dt(dt, WOt, d, h * dh, src, bO, out, B, kh_max * dh, 0, status, st));
}

int wbytes_of(dv_dtype t) { return t == DV_BF16 ? 2 : 4; }
bool dtype_ok(int t) { return t == DV_F32 || t == DV_BF16; }
bool mode_ok(int m) { return m == DV_TOPK || m == DV_THRESHOLD; }
bool act_ok(int a) { return a == DV_ACT_RELU || a == DV_ACT_GELU; }

dv_status check_ws(const Layout& L, void* ws, size_t ws_bytes) {
  if (!ok_ptr(ws)) return ws ? DV_ERR_ALIGN : DV_ERR_ARG;
  if (ws_bytes < L.total) return DV_ERR_WORKSPACE;
  return DV_OK;
}

// ---------------------------------------------------------------------------
// Tensor-core path (dv_tc.cuh) for batch 5..16 with bf16 weights
// ---------------------------------------------------------------------------

bool tc_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("DV_TC");
    return !(e && e[0] == '0');
  }();
  return on;
}

// Batch 5-16, and batch 3-4 when the rows are too long for the column-owner
// kernels (d > 4096 bf16), where the CUDA-core row kernels would take them.
bool tc_ok(int B, int d, dv_dtype wdt, int dh, int k_max) {
  const bool batch = B >= TC_MIN_B || (B >= 3 && !co_ok(B, d, 8));
  return tc_enabled() && batch && tc_shape_ok(B, d, wbytes_of(wdt), dh > 0 ? dh : 64, k_max);
}

dv_status tc_mlp(const Layout& L, void* ws, const float* y, int B, int d, int N, const void* W1t, const float* b1,
                 const void* W2t, const float* b2, const int32_t* idx, const int32_t* count, int k_max, float* out,
                 int act, cudaStream_t st) {
  TcMlpArgs a = {};
  a.act = act;
  a.W1t = static_cast<const bf16*>(W1t);
  a.b1 = b1;
  a.W2t = static_cast<const bf16*>(W2t);
  a.b2 = b2;
  a.idx = idx;
  a.count = count;
  a.k_max = k_max;
  a.d = d;
  a.N = N;
  a.nb = B;
  a.KC = L.KC;
  bf16* xhi = at<bf16>(ws, L.tc_x);
  a.xhi = xhi;
  a.xlo = xhi + (size_t)TC_N * L.XC;
  a.act_hi = at<bf16>(ws, L.tc_act);
  a.act_lo = a.act_hi + (size_t)TC_N * (L.KC > 0 ? L.KC : 1);
  a.rowid_c = at<int32_t>(ws, L.tc_rowid);
  a.tile_cnt = at<int32_t>(ws, L.tc_tiles);
  a.red = at<float>(ws, L.tc_red);
  a.tick = at<unsigned>(ws, L.tc_tick);
  a.acc = at<unsigned long long>(ws, L.tc_acc);
  a.out = out;
  a.status = at<int>(ws, L.status);
  if (k_max > 0) DV_TRY(run_tc_split(y, B, d, d, xhi, xhi + (size_t)TC_N * L.XC, d, st));
  return cuda_status(run_tc_mlp(a, st));
}

dv_status tc_qkv(const Layout& L, void* ws, const float* y, int B, int d, int h, int dh, const void* Wqkv,
                 const float* bqkv, void* Kc, void* Vc, int cap, int pos, const int32_t* head_idx,
                 const int32_t* head_count, int kh_max, cudaStream_t st) {
  TcQkvArgs a = {};
  a.Wqkv = static_cast<const bf16*>(Wqkv);
  a.bqkv = bqkv;
  bf16* xhi = at<bf16>(ws, L.tc_x);
  a.xhi = xhi;
  a.xlo = xhi + (size_t)TC_N * L.XC;
  a.head_idx = head_idx;
  a.head_count = head_count;
  a.kh_max = kh_max;
  a.h = h;
  a.dh = dh;
  a.d = d;
  a.nb = B;
  a.cap = cap;
  a.pos = pos;
  a.q = at<float>(ws, L.q);
  a.Kc = static_cast<bf16*>(Kc);
  a.Vc = static_cast<bf16*>(Vc);
  a.status = at<int>(ws, L.status);
  a.red = at<float>(ws, L.tc_red);
  a.tick = at<unsigned>(ws, L.tc_tick);
  DV_TRY(run_tc_split(y, B, d, d, xhi, xhi + (size_t)TC_N * L.XC, d, st));
  return cuda_status(run_tc_qkv(a, st));
}

dv_status tc_wo(const Layout& L, void* ws, int B, int d, int h, int dh, const void* WOt, const float* bO,
                const int32_t* head_idx, const int32_t* head_count, int kh_max, float* out, cudaStream_t st) {
  TcWoArgs a = {};
  a.WOt = static_cast<const bf16*>(WOt);
  a.bO = bO;
  bf16* hhi = at<bf16>(ws, L.tc_x);
  a.hhi = hhi;
  a.hlo = hhi + (size_t)TC_N * L.XC;
  a.head_idx = head_idx;
  a.head_count = head_count;
  a.kh_max = kh_max;
  a.h = h;
  a.dh = dh;
  a.d = d;
  a.nb = B;
  a.out = out;
  a.status = at<int>(ws, L.status);
  a.acc = at<unsigned long long>(ws, L.tc_acc);
  if (kh_max > 0)
    DV_TRY(run_tc_split(at<float>(ws, L.H), B, kh_max * dh, (long long)kh_max * dh, hhi, hhi + (size_t)TC_N * L.XC,
                        (long long)kh_max * dh, st));
  return cuda_status(run_tc_wo(a, st));
}

// ---------------------------------------------------------------------------
// Fused layer path (dv_fused.cuh)
// ---------------------------------------------------------------------------


bool fused_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("DV_FUSED");
    return !(e && e[0] == '0');
  }();
  return on;
}

// Shapes the fused kernels take: column slices of W^O whole 16-byte vectors,
// the normalised input and the K/V tiles within shared memory.
bool fused_ok(const dv_dims& D, dv_dtype wdt) {
  if (!fused_enabled()) return false;
  if (tc_ok(D.B, D.d, wdt, D.dh, D.k_max)) return false;  // batch 5..16, bf16: tensor-core kernels
  const int wb = wbytes_of(wdt), E = 16 / wb;
  if (D.d % (ATTN_CS * E) != 0) return false;
  if ((size_t)D.B * D.d * 4 > 160 * 1024) return false;
  if (attn_out_smem(attn_out_S(D.cap - 1), D.dh, wb, D.B) > ATTN_SMEM_MAX) return false;
  if (D.N > SEL_SMEM_KEYS || D.h > HSEL_MAX) return false;
  return true;
}


// Second half of the fused predictor: neuron scores from z (in ws) and the
// selections; the head scores sh must be complete when heads is set.
// The smallest batch whose look-ahead neuron scores z B^T + b1 run on the
// tensor cores (tc_dense_kernel) in the fused path; below it predict_b_kernel
// (DV_PB_TC_MIN_B overrides; 17 keeps predict_b_kernel at every batch). At
// the OPT-175B shape the tensor-core form made the look-ahead step faster at
// batch 1 (106.2 against 110.0 us per layer) and batch 2 (212.2 against
// 247.2), although alone it is no faster at batch 1 (49.7 against 46.9 us
// with the selection): its CTAs share the SMs with the main kernels better.
int pb_tc_min_batch() {
  static const int b = [] {
    const char* e = std::getenv("DV_PB_TC_MIN_B");
    const int v = e ? std::atoi(e) : 0;
    return v > 0 ? v : 1;
  }();
  return b;
}

dv_status fused_predict_rest(const Layout& L, void* ws, const dv_layer_weights* w, const dv_dims& D,
                             const dv_layer_params* p, bool heads, bool neurons, float* sh, int32_t* hidx,
                             int32_t* hcnt, float* sm, int32_t* midx, int32_t* mcnt, cudaStream_t st) {
  if (neurons) {
    // large predictors only: at the OPT-1.3B and OPT-6.7B shapes (B of 4 and
    // 17 MB) the tensor-core form made the step slower (by 2-6 and 1 us per
    // layer); from the OPT-66B shape (75 MB) on it made it faster
    const bool large = (long long)D.N * D.r >= (16ll << 20);
    if (large && D.B >= pb_tc_min_batch() && tc_enabled() && tc_dense_ok(D.B, wbytes_of(w->wdtype), D.N, D.r)) {
      DV_TRY(pred_tc(L, ws, w->Bm, D.N, D.r, w->b1, at<float>(ws, L.z), D.B, sm, D.N, st));
    } else {
      PredictBArgs b = {};
      b.z = at<float>(ws, L.z);
      b.Bm = w->Bm;
      b.b1 = w->b1;
      b.N = D.N;
      b.r = D.r;
      b.nb = D.B;
      b.scores = sm;
      DV_TRY(run_predict_b_dt(w->wdtype, b, st));
    }
    DV_TRY(select_any(sm, D.B, D.N, p->k, p->tau, p->mode, at<uint32_t>(ws, L.bm_m), at<unsigned>(ws, L.pb_ticket),
                      midx, mcnt, st));
  }
  if (heads) {
    SelectHeadsArgs f{sh, D.B, D.h, p->k_h, p->mode_h, p->tau_h, hidx, hcnt};
    const size_t smem = 4ull * D.h;
    DV_TRY(allow_smem(select_heads_kernel, smem));
    DV_TRY(launch(select_heads_kernel, dim3(1), dim3(SEL_THREADS), smem, st, f));
  }
  return DV_OK;
}

// The head set (heads) and/or the neuron set (neurons) predicted from y:
// predict_a (head scores, z = y A), predict_b (neuron scores), then the exact
// top-k / threshold selections (select_rows_kernel for the neurons,
// select_heads_kernel for the heads).
dv_status fused_predict(const Layout& L, void* ws, const dv_layer_weights* w, const dv_dims& D,
                        const dv_layer_params* p, const float* y, bool heads, bool neurons, float* sh, int32_t* hidx,
                        int32_t* hcnt, float* sm, int32_t* midx, int32_t* mcnt, cudaStream_t st) {
  PredictAArgs a = {};
  a.y = y;
  a.PA = heads ? w->PA : nullptr;
  a.At = neurons ? w->At : nullptr;
  a.h = D.h;
  a.r = D.r;
  a.d = D.d;
  a.nb = D.B;
  a.scores_h = sh;
  a.z = at<float>(ws, L.z);
  DV_TRY(run_predict_a_any_dt(w->wdtype, a, st));
  return fused_predict_rest(L, ws, w, D, p, heads, neurons, sh, hidx, hcnt, sm, midx, mcnt, st);
}

// Pointers a layer call writes: the trace buffers when given, else workspace.
struct LayerBufs {
  float *yA, *yM, *sh, *sm;
  int32_t *hidx, *hcnt, *midx, *mcnt;
  const int32_t *use_hidx, *use_hcnt, *use_midx, *use_mcnt;
};

LayerBufs layer_bufs(const Layout& L, void* ws, const dv_layer_io* sel, const dv_layer_io* trace) {
  const dv_layer_io none = {};
  const dv_layer_io& t = trace ? *trace : none;
  LayerBufs r;
  r.yA = t.yA ? t.yA : at<float>(ws, L.yA);
  r.yM = t.yM ? t.yM : at<float>(ws, L.yM);
  r.sh = t.scores_h ? t.scores_h : at<float>(ws, L.scores_h);
  r.hidx = t.head_idx ? t.head_idx : at<int32_t>(ws, L.head_idx);
  r.hcnt = t.head_count ? t.head_count : at<int32_t>(ws, L.head_count);
  r.sm = t.scores ? t.scores : at<float>(ws, L.scores);
  r.midx = t.idx ? t.idx : at<int32_t>(ws, L.idx);
  r.mcnt = t.count ? t.count : at<int32_t>(ws, L.count);
  r.use_hidx = sel ? sel->head_idx : r.hidx;
  r.use_hcnt = sel ? sel->head_count : r.hcnt;
  r.use_midx = sel ? sel->idx : r.midx;
  r.use_mcnt = sel ? sel->count : r.mcnt;
  return r;
}

// First half of a layer: LN1, the head set unless given, Q/K/V + KV append.
// The first half of the next layer's look-ahead predictor, computed with a
// layer's q, k, v: head scores into sh, z into z.
struct Ahead {
  const dv_layer_weights* w;
  float* sh;
  float* z;
};

dv_status layer_begin_fused_qkv(const dv_layer_weights* w, const dv_dims& D, AttnInArgs a, const Ahead* ahead,
                                float* yA_ws, cudaStream_t st);

dv_status layer_begin(const Layout& L, void* ws, const dv_layer_weights* w, const dv_dims& D, const dv_layer_params* p,
                      float* x, int pos, const dv_layer_io* sel, const dv_layer_io* trace, cudaStream_t st,
                      const Ahead* ahead = nullptr) {
  const LayerBufs r = layer_bufs(L, ws, sel, trace);
  int* status = at<int>(ws, L.status);
  if (ahead && !fused_ok(D, w->wdtype)) {
    // kernel-per-step path: the layer, then the two predictor GEMVs from yA
    float* yA = (sel && sel->yA) ? sel->yA : r.yA;
    dv_layer_io tr = trace ? *trace : dv_layer_io{};
    if (!(sel && sel->yA)) tr.yA = yA;
    DV_CHECK(layer_begin(L, ws, w, D, p, x, pos, sel, &tr, st));
    if (!fused_enabled()) {
      DV_TRY(run_gemv(w->wdtype, ahead->w->PA, D.h, D.d, yA, D.d, D.B, nullptr, ahead->sh, D.h, st));
      return cuda_status(run_gemv(w->wdtype, ahead->w->At, D.r, D.d, yA, D.d, D.B, nullptr, ahead->z, D.r, st));
    }
    const bool tc_h = pred_tc_ok(D.B, w->wdtype, D.h, D.d), tc_z = pred_tc_ok(D.B, w->wdtype, D.r, D.d);
    if (tc_h && tc_z) {  // head scores and z in one launch: rows of P_A, then rows of A^T
      bf16* xhi = at<bf16>(ws, L.tc_x);
      bf16* xlo = xhi + (size_t)TC_N * L.XC;
      DV_TRY(run_tc_split(yA, D.B, D.d, D.d, xhi, xlo, D.d, st));
      return cuda_status(run_tc_dense(static_cast<const bf16*>(ahead->w->PA), D.h, nullptr, ahead->sh, D.h,
                                      static_cast<const bf16*>(ahead->w->At), D.r, nullptr, ahead->z, D.r, D.d, xhi,
                                      xlo, D.B, at<float>(ws, L.tc_red), at<unsigned>(ws, L.tc_tick), status, st));
    }
    if (tc_h) DV_TRY(pred_tc(L, ws, ahead->w->PA, D.h, D.d, nullptr, yA, D.B, ahead->sh, D.h, st));
    if (tc_z) DV_TRY(pred_tc(L, ws, ahead->w->At, D.r, D.d, nullptr, yA, D.B, ahead->z, D.r, st, !tc_h));
    PredictAArgs pa = {};
    pa.y = yA;
    pa.PA = tc_h ? nullptr : ahead->w->PA;
    pa.At = tc_z ? nullptr : ahead->w->At;
    pa.h = D.h;
    pa.r = D.r;
    pa.d = D.d;
    pa.nb = D.B;
    pa.scores_h = ahead->sh;
    pa.z = ahead->z;
    return cuda_status(run_predict_a_any_dt(w->wdtype, pa, st));
  }
  if (fused_ok(D, w->wdtype)) {
    if (!sel) {
      DV_TRY(launch(layernorm_kernel, dim3(D.B), LN_THREADS, 0, st, (const float*)x, r.yA, D.d, w->ln1_g, w->ln1_b,
                    p->eps));
      DV_CHECK(fused_predict(L, ws, w, D, p, r.yA, true, false, r.sh, r.hidx, r.hcnt, nullptr, nullptr, nullptr, st));
    }
    AttnInArgs a = {};
    a.x = x;
    a.t1 = at<float>(ws, L.t1);
    a.yA_out = sel ? (trace ? trace->yA : nullptr) : nullptr;
    a.ln_g = w->ln1_g;
    a.ln_b = w->ln1_b;
    a.eps = p->eps;
    a.Wqkv = w->Wqkv;
    a.bqkv = w->bqkv;
    a.head_idx = r.use_hidx;
    a.head_count = r.use_hcnt;
    a.kh_max = D.kh_max;
    a.q = at<float>(ws, L.q);
    a.Kc = w->Kc;
    a.Vc = w->Vc;
    a.h = D.h;
    a.dh = D.dh;
    a.d = D.d;
    a.cap = D.cap;
    a.pos = pos;
    a.nb = D.B;
    a.sets_ready = sel ? 1 : 0;
    a.status = status;
    if (p->exact_kv && !a.yA_out) a.yA_out = r.yA;  // the other heads' k, v are formed from yA
    DV_CHECK(layer_begin_fused_qkv(w, D, a, ahead, r.yA, st));
    if (p->exact_kv)
      DV_TRY(run_kv_rest_dt(w->wdtype, w->Wqkv, D.d, D.h, D.dh, a.yA_out, D.B, w->bqkv, r.use_hidx, r.use_hcnt,
                            D.kh_max, w->Kc, w->Vc, D.cap, pos, status, st));
    return DV_OK;
  }
  // kernel-per-step path
  float* yA = r.yA;
  if (sel && sel->yA) {
    yA = sel->yA;  // LN1(x) computed by the caller
  } else {
    DV_TRY(launch(layernorm_kernel, dim3(D.B), LN_THREADS, 0, st, (const float*)x, yA, D.d, w->ln1_g, w->ln1_b,
                  p->eps));
  }
  if (!sel)
    DV_CHECK(do_predict_heads(L, ws, yA, D.B, D.d, D.h, w->PA, w->wdtype, p->k_h, p->tau_h, p->mode_h, r.sh, r.hidx,
                              r.hcnt, st));
  if (D.kh_max > 0) {
    if (tc_ok(D.B, D.d, w->wdtype, D.dh, D.k_max)) {
      DV_CHECK(tc_qkv(L, ws, yA, D.B, D.d, D.h, D.dh, w->Wqkv, w->bqkv, w->Kc, w->Vc, D.cap, pos, r.use_hidx,
                      r.use_hcnt, D.kh_max, st));
    } else {
      DV_TRY(run_qkv_dt(w->wdtype, w->Wqkv, D.d, D.h, D.dh, yA, D.B, w->bqkv, r.use_hidx, r.use_hcnt, D.kh_max,
                        at<float>(ws, L.q), w->Kc, w->Vc, D.cap, pos, status, st));
    }
  }
  if (p->exact_kv)
    DV_TRY(run_kv_rest_dt(w->wdtype, w->Wqkv, D.d, D.h, D.dh, yA, D.B, w->bqkv, r.use_hidx, r.use_hcnt, D.kh_max, w->Kc,
                          w->Vc, D.cap, pos, status, st));
  return DV_OK;
}

// The fused Q/K/V launch of layer_begin (a filled in), with the next
// layer's predictor first stage when `ahead` is given; yA_ws receives LN1(x)
// when the first stage needs its own launch.
dv_status layer_begin_fused_qkv(const dv_layer_weights* w, const dv_dims& D, AttnInArgs a, const Ahead* ahead,
                                float* yA_ws, cudaStream_t st) {
  if (ahead && attn_in_takes_rows(D.B, D.d, w->wdtype == DV_BF16 ? 8 : 4)) {
    a.PA2 = ahead->w->PA;
    a.At2 = ahead->w->At;
    a.sh2 = ahead->sh;
    a.z2 = ahead->z;
    a.n2h = D.h;
    a.n2r = D.r;
    return cuda_status(run_attn_in_any_dt(w->wdtype, a, st));
  }
  if (ahead) {  // the row kernel: the predictor's first stage as its own launch, from yA
    if (!a.yA_out) a.yA_out = yA_ws;
    DV_TRY(run_attn_in_any_dt(w->wdtype, a, st));
    PredictAArgs pa = {};
    pa.y = a.yA_out;
    pa.PA = ahead->w->PA;
    pa.At = ahead->w->At;
    pa.h = D.h;
    pa.r = D.r;
    pa.d = D.d;
    pa.nb = D.B;
    pa.scores_h = ahead->sh;
    pa.z = ahead->z;
    return cuda_status(run_predict_a_any_dt(w->wdtype, pa, st));
  }
  return cuda_status(run_attn_in_any_dt(w->wdtype, a, st));
}

// Attention half: split attention over the selected heads, W^O, residual.
dv_status layer_attn(const Layout& L, void* ws, const dv_layer_weights* w, const dv_dims& D, const dv_layer_params* p,
                     float* x, int pos, const dv_layer_io* sel, const dv_layer_io* trace, cudaStream_t st) {
  const LayerBufs r = layer_bufs(L, ws, sel, trace);
  int* status = at<int>(ws, L.status);
  if (fused_ok(D, w->wdtype)) {
    AttnOutArgs b = {};
    b.q = at<float>(ws, L.q);
    b.Kc = w->Kc;
    b.Vc = w->Vc;
    b.WOt = w->WOt;
    b.bO = w->bO;
    b.head_idx = r.use_hidx;
    b.head_count = r.use_hcnt;
    b.kh_max = D.kh_max;
    b.x = x;
    b.t1 = at<float>(ws, L.t1);
    b.h = D.h;
    b.dh = D.dh;
    b.d = D.d;
    b.cap = D.cap;
    b.pos = pos;
    b.nb = D.B;
    b.S = attn_out_S(pos);
    b.sets_ready = sel ? 1 : 0;
    b.scale = p->scale;
    b.status = status;
    const int E = w->wdtype == DV_BF16 ? 8 : 4;
    if (w->wdtype == DV_BF16 && wo_split_ok(D.B, D.d, E, wbytes_of(w->kvdtype))) {
      b.H_out = at<float>(ws, L.H);  // attention only; then the W^O rows over every SM
      DV_TRY(run_attn_out_dt(w->kvdtype, b, st));
      WoStreamArgs o = {};
      o.WOt = w->WOt;
      o.bO = w->bO;
      o.H = b.H_out;
      o.head_idx = r.use_hidx;
      o.head_count = r.use_hcnt;
      o.kh_max = D.kh_max;
      o.h = D.h;
      o.dh = D.dh;
      o.d = D.d;
      o.nb = D.B;
      o.sets_ready = b.sets_ready;
      o.x = x;
      o.t1 = b.t1;
      o.status = status;
      return cuda_status(run_wo_stream_dt(w->wdtype, o, st));
    }
    return cuda_status(run_attn_out_dt(w->kvdtype, b, st));
  }
  if (tc_ok(D.B, D.d, w->wdtype, D.dh, D.k_max)) {
    if (D.kh_max > 0)
      DV_TRY(run_attn_dt(w->kvdtype, D.dh, at<float>(ws, L.q), w->Kc, w->Vc, D.B, D.h, D.cap, pos, p->scale,
                         r.use_hidx, r.use_hcnt, D.kh_max, at<float>(ws, L.part), at<unsigned>(ws, L.attn_ctr),
                         at<float>(ws, L.H), status, st));
    return tc_wo(L, ws, D.B, D.d, D.h, D.dh, w->WOt, w->bO, r.use_hidx, r.use_hcnt, D.kh_max, x, st);
  }
  if (D.kh_max > 0) {
    float* H = at<float>(ws, L.H);
    const float* q = at<float>(ws, L.q);
    DV_TRY(run_attn_dt(w->kvdtype, D.dh, q, w->Kc, w->Vc, D.B, D.h, D.cap, pos, p->scale, r.use_hidx, r.use_hcnt, D.kh_max, at<float>(ws, L.part), at<unsigned>(ws, L.attn_ctr), H, status, st));
    RowsHeads src{r.use_hidx, r.use_hcnt, H, D.kh_max, D.dh, D.h};
    return cuda_status(run_axpy_dt(w->wdtype, w->WOt, D.d, D.h * D.dh, src, w->bO, x, D.B, D.kh_max * D.dh, 0, status, st));
  }
  if (w->bO) {
    RowsHeads none{r.use_hidx, r.use_hcnt, nullptr, 0, D.dh, D.h};
    return cuda_status(run_axpy_dt(w->wdtype, w->WOt, D.d, D.h * D.dh, none, w->bO, x, D.B, 1, 0, status, st));
  }
  return DV_OK;
}

// MLP half: LN2, the neuron set unless given, the sparse MLP + residual.
dv_status layer_mlp(const Layout& L, void* ws, const dv_layer_weights* w, const dv_dims& D, const dv_layer_params* p,
                    float* x, const dv_layer_io* sel, const dv_layer_io* trace, cudaStream_t st) {
  const LayerBufs r = layer_bufs(L, ws, sel, trace);
  int* status = at<int>(ws, L.status);
  if (fused_ok(D, w->wdtype)) {
    float* t1 = at<float>(ws, L.t1);
    if (!sel) {
      DV_TRY(launch(layernorm_kernel, dim3(D.B), LN_THREADS, 0, st, (const float*)t1, r.yM, D.d, w->ln2_g, w->ln2_b,
                    p->eps));
      DV_CHECK(fused_predict(L, ws, w, D, p, r.yM, false, true, nullptr, nullptr, nullptr, r.sm, r.midx, r.mcnt, st));
    }
    MlpBlockArgs c = {};
    c.t1 = t1;
    c.x = x;
    c.ln_g = w->ln2_g;
    c.ln_b = w->ln2_b;
    c.eps = p->eps;
    c.W1t = w->W1t;
    c.b1 = w->b1;
    c.W2t = w->W2t;
    c.b2 = w->b2;
    c.idx = r.use_midx;
    c.count = r.use_mcnt;
    c.k_max = D.k_max;
    c.d = D.d;
    c.N = D.N;
    c.nb = D.B;
    c.G = mlp_block_grid(D.k_max);
    c.sets_ready = sel ? 1 : 0;
    c.yM_out = sel ? (trace ? trace->yM : nullptr) : nullptr;
    c.status = status;
    c.act = p->act;
    return cuda_status(run_mlp_block_any_dt(w->wdtype, c, st));
  }
  DV_TRY(launch(layernorm_kernel, dim3(D.B), LN_THREADS, 0, st, (const float*)x, r.yM, D.d, w->ln2_g, w->ln2_b,
                p->eps));
  if (!sel)
    DV_CHECK(do_predict_mlp(L, ws, r.yM, D.B, D.d, D.r, D.N, w->At, w->Bm, w->b1, w->wdtype, p->k, p->tau, p->mode,
                            r.sm, r.midx, r.mcnt, st));
  return do_sparse_mlp(L, ws, r.yM, D.B, D.d, D.N, w->W1t, w->b1, w->W2t, w->b2, w->wdtype, r.use_midx, r.use_mcnt,
                       D.k_max, x, 1, p->act, st);
}

dv_status layer_end(const Layout& L, void* ws, const dv_layer_weights* w, const dv_dims& D, const dv_layer_params* p,
                    float* x, int pos, const dv_layer_io* sel, const dv_layer_io* trace, cudaStream_t st) {
  DV_CHECK(layer_attn(L, ws, w, D, p, x, pos, sel, trace, st));
  return layer_mlp(L, ws, w, D, p, x, sel, trace, st);
}

}  // namespace

// ===========================================================================
// Public entry points
// ===========================================================================

extern "C" {

uint64_t dv_launch_count(void) { return g_launches.load(); }

const char* dv_status_string(dv_status s) {
  switch (s) {
    case DV_OK: return "ok";
    case DV_ERR_ARG: return "invalid argument";
    case DV_ERR_ALIGN: return "pointer not 16-byte aligned";
    case DV_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case DV_ERR_CUDA: return "CUDA error";
    case DV_ERR_DEVICE: return "device status word set";
    case DV_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

size_t dv_workspace_size(int op, const dv_dims* dims) {
  if (!dims || op < DV_OP_PREDICT_MLP || op > DV_OP_DECODE_LAYER) return 0;
  dv_dims D = *dims;
  if (op == DV_OP_TOPK) {
    D.d = 8;
    D.r = 0;
    D.h = 0;
    D.dh = 0;
    D.cap = 0;
    D.kh_max = 0;
  }
  if (!dims_ok(D)) return 0;
  size_t n = 0;
  for (int wb : {1, 2, 4}) n = layout(D, wb).total > n ? layout(D, wb).total : n;  // int8, bf16, fp32 weights
  return n;
}

dv_status dv_read_device_status(void* ws, dv_stream_t stream, int* out) {
  if (!ws || !out) return DV_ERR_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  DV_TRY(cudaStreamSynchronize(st));
  DV_TRY(cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost));
  DV_TRY(cudaMemset(ws, 0, sizeof(int)));
  *out = v;
  return DV_OK;
}

dv_status dv_predict_mlp(const float* y, int B, int d, int r, int N, const void* At, const void* Bm, const float* b1,
                         dv_dtype wdtype, int k, float tau, int mode, float* scores, int32_t* idx, int32_t* count,
                         void* ws, size_t ws_bytes, dv_stream_t stream) {
  if (!dtype_ok(wdtype) || !mode_ok(mode)) return DV_ERR_ARG;
  if (!y || !At || !Bm || !b1 || !scores || !idx || !count) return DV_ERR_ARG;
  if (!ok_ptr(y) || !ok_ptr(At) || !ok_ptr(Bm) || !ok_ptr(b1) || !ok_ptr(scores)) return DV_ERR_ALIGN;
  dv_dims D = {B, d, N, r, 0, 0, 0, (k > N ? N : (k < 0 ? 0 : k)), 0};
  if (!dims_ok(D) || r < 8) return DV_ERR_ARG;
  const Layout L = layout(D, wbytes_of(wdtype));
  DV_CHECK(check_ws(L, ws, ws_bytes));
  return do_predict_mlp(L, ws, y, B, d, r, N, At, Bm, b1, wdtype, k, tau, mode, scores, idx, count,
                        reinterpret_cast<cudaStream_t>(stream));
}

dv_status dv_predict_heads(const float* y, int B, int d, int h, const void* PA, dv_dtype wdtype, int k_h, float tau,
                           int mode, float* scores, int32_t* head_idx, int32_t* head_count, void* ws, size_t ws_bytes,
                           dv_stream_t stream) {
  if (!dtype_ok(wdtype) || !mode_ok(mode)) return DV_ERR_ARG;
  if (!y || !PA || !scores || !head_idx || !head_count || h < 1) return DV_ERR_ARG;
  if (!ok_ptr(y) || !ok_ptr(PA)) return DV_ERR_ALIGN;
  dv_dims D = {B, d, 1, 0, h, 8, 0, 0, (k_h > h ? h : (k_h < 0 ? 0 : k_h))};
  if (!dims_ok(D)) return DV_ERR_ARG;
  const Layout L = layout(D, wbytes_of(wdtype));
  DV_CHECK(check_ws(L, ws, ws_bytes));
  return do_predict_heads(L, ws, y, B, d, h, PA, wdtype, k_h, tau, mode, scores, head_idx, head_count,
                          reinterpret_cast<cudaStream_t>(stream));
}

dv_status dv_topk(const float* scores, int B, int n, int k, float tau, int mode, int32_t* idx, int32_t* count,
                  void* ws, size_t ws_bytes, dv_stream_t stream) {
  if (!mode_ok(mode) || !scores || !idx || !count || n < 1 || B < 1 || B > 16) return DV_ERR_ARG;
  if (!ok_ptr(scores)) return DV_ERR_ALIGN;
  dv_dims D = {B, 8, n, 0, 0, 0, 0, (k > n ? n : (k < 0 ? 0 : k)), 0};
  const Layout L = layout(D, 2);
  DV_CHECK(check_ws(L, ws, ws_bytes));
  return cuda_status(select_any(scores, B, n, k, tau, mode, at<uint32_t>(ws, L.bm_m), at<unsigned>(ws, L.sel_ticket_m),
                                idx, count, reinterpret_cast<cudaStream_t>(stream)));
}

dv_status dv_sparse_mlp_act(const float* y, int B, int d, int N, const void* W1t, const float* b1, const void* W2t,
                            const float* b2, dv_dtype wdtype, const int32_t* idx, const int32_t* count, int k_max,
                            float* out, int accumulate, int act, void* ws, size_t ws_bytes, dv_stream_t stream) {
  if (!dtype_ok(wdtype) || !act_ok(act)) return DV_ERR_ARG;
  if (!y || !W1t || !b1 || !W2t || !idx || !count || !out) return DV_ERR_ARG;
  if (!ok_ptr(y) || !ok_ptr(W1t) || !ok_ptr(W2t) || !ok_ptr(out) || !ok_opt(b2)) return DV_ERR_ALIGN;
  dv_dims D = {B, d, N, 0, 0, 0, 0, k_max, 0};
  if (!dims_ok(D)) return DV_ERR_ARG;
  const Layout L = layout(D, wbytes_of(wdtype));
  DV_CHECK(check_ws(L, ws, ws_bytes));
  return do_sparse_mlp(L, ws, y, B, d, N, W1t, b1, W2t, b2, wdtype, idx, count, k_max, out, accumulate, act,
                       reinterpret_cast<cudaStream_t>(stream));
}

dv_status dv_sparse_mlp(const float* y, int B, int d, int N, const void* W1t, const float* b1, const void* W2t,
                        const float* b2, dv_dtype wdtype, const int32_t* idx, const int32_t* count, int k_max,
                        float* out, int accumulate, void* ws, size_t ws_bytes, dv_stream_t stream) {
  return dv_sparse_mlp_act(y, B, d, N, W1t, b1, W2t, b2, wdtype, idx, count, k_max, out, accumulate, DV_ACT_RELU, ws,
                           ws_bytes, stream);
}

dv_status dv_sparse_mha(const float* y, int B, int d, int h, int dh, const void* Wqkv, const float* bqkv,
                        const void* WOt, const float* bO, dv_dtype wdtype, void* Kc, void* Vc, dv_dtype kvdtype,
                        int cap, int pos, float scale, const int32_t* head_idx, const int32_t* head_count, int kh_max,
                        float* out, int accumulate, void* ws, size_t ws_bytes, dv_stream_t stream) {
  if (!dtype_ok(wdtype) || !dtype_ok(kvdtype)) return DV_ERR_ARG;
  if (kvdtype != wdtype) return DV_ERR_UNSUPPORTED;
  if (!y || !Wqkv || !WOt || !Kc || !Vc || !head_idx || !head_count || !out) return DV_ERR_ARG;
  if (!ok_ptr(y) || !ok_ptr(Wqkv) || !ok_ptr(WOt) || !ok_ptr(Kc) || !ok_ptr(Vc) || !ok_ptr(out) || !ok_opt(bO))
    return DV_ERR_ALIGN;
  if (dh != 64 && dh != 128) return DV_ERR_UNSUPPORTED;
  if (cap < 1 || pos < 0 || pos >= cap) return DV_ERR_ARG;
  dv_dims D = {B, d, 1, 0, h, dh, cap, 0, kh_max};
  if (!dims_ok(D) || h < 1) return DV_ERR_ARG;
  const Layout L = layout(D, wbytes_of(wdtype));
  DV_CHECK(check_ws(L, ws, ws_bytes));
  return do_sparse_mha(L, ws, y, B, d, h, dh, Wqkv, bqkv, WOt, bO, wdtype, Kc, Vc, cap, pos, scale, head_idx,
                       head_count, kh_max, out, accumulate, reinterpret_cast<cudaStream_t>(stream));
}

dv_status dv_sparse_mlp_q8(const float* y, int B, int d, int N, const int8_t* W1q, const float* W1s, const float* b1,
                           const int8_t* W2q, const float* W2s, const float* b2, const int32_t* idx,
                           const int32_t* count, int k_max, float* out, int accumulate, int act, void* ws,
                           size_t ws_bytes, dv_stream_t stream) {
  if (!act_ok(act)) return DV_ERR_ARG;
  if (!y || !W1q || !W1s || !b1 || !W2q || !W2s || !idx || !count || !out) return DV_ERR_ARG;
  if (!ok_ptr(y) || !ok_ptr(W1q) || !ok_ptr(W2q) || !ok_ptr(W1s) || !ok_ptr(W2s) || !ok_ptr(out) || !ok_opt(b2))
    return DV_ERR_ALIGN;
  dv_dims D = {B, d, N, 0, 0, 0, 0, k_max, 0};
  if (!dims_ok(D)) return DV_ERR_ARG;
  if (B > 4 || d % 16 != 0) return DV_ERR_UNSUPPORTED;
  const Layout L = layout(D, 1);
  DV_CHECK(check_ws(L, ws, ws_bytes));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!accumulate) DV_TRY(cudaMemsetAsync(out, 0, 4ull * B * d, st));
  int* status = at<int>(ws, L.status);
  if (L.nseg == 0) {
    if (b2) {  // nothing selected: out (+)= b2 only
      RowsHeads none{idx, count, nullptr, 0, 1, 0};
      return cuda_status(run_axpy_q8(W2q, d, N, none, b2, out, B, 1, 0, status, st));
    }
    return DV_OK;
  }
  int32_t* seg_idx = at<int32_t>(ws, L.seg_idx);
  float* seg_a = at<float>(ws, L.seg_a);
  int32_t* seg_cnt = at<int32_t>(ws, L.seg_cnt);
  DV_TRY(run_mlp_up_q8(W1q, W1s, d, N, y, B, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, L.nseg, act, st));
  RowsMlp src{seg_idx, seg_a, seg_cnt, L.nseg, L.SEG, W2s};
  return cuda_status(run_axpy_q8(W2q, d, N, src, b2, out, B, k_max, 4ull * (L.nseg + 1), status, st));
}

dv_status dv_sparse_mha_q8(const float* y, int B, int d, int h, int dh, const int8_t* Wqkvq, const float* Wqkv_s,
                           const float* bqkv, const int8_t* WOq, const float* WO_s, const float* bO, void* Kc, void* Vc,
                           int cap, int pos, float scale, const int32_t* head_idx, const int32_t* head_count,
                           int kh_max, float* out, int accumulate, void* ws, size_t ws_bytes, dv_stream_t stream) {
  if (!y || !Wqkvq || !Wqkv_s || !WOq || !WO_s || !Kc || !Vc || !head_idx || !head_count || !out) return DV_ERR_ARG;
  if (!ok_ptr(y) || !ok_ptr(Wqkvq) || !ok_ptr(Wqkv_s) || !ok_ptr(WOq) || !ok_ptr(WO_s) || !ok_ptr(Kc) ||
      !ok_ptr(Vc) || !ok_ptr(out) || !ok_opt(bO) || !ok_opt(bqkv))
    return DV_ERR_ALIGN;
  if (dh != 64 && dh != 128) return DV_ERR_UNSUPPORTED;
  if (cap < 1 || pos < 0 || pos >= cap) return DV_ERR_ARG;
  dv_dims D = {B, d, 1, 0, h, dh, cap, 0, kh_max};
  if (!dims_ok(D) || h < 1) return DV_ERR_ARG;
  if (B > 4 || d % 16 != 0) return DV_ERR_UNSUPPORTED;
  const Layout L = layout(D, 1);
  DV_CHECK(check_ws(L, ws, ws_bytes));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!accumulate) DV_TRY(cudaMemsetAsync(out, 0, 4ull * B * d, st));
  int* status = at<int>(ws, L.status);
  if (kh_max == 0) {
    if (bO) {
      RowsHeads none{head_idx, head_count, nullptr, 0, dh, h};
      return cuda_status(run_axpy_q8(WOq, d, h * dh, none, bO, out, B, 1, 0, status, st));
    }
    return DV_OK;
  }
  float* q = at<float>(ws, L.q);
  float* H = at<float>(ws, L.H);
  DV_TRY(run_qkv_q8(Wqkvq, Wqkv_s, d, h, dh, y, B, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos, status,
                    st));
  DV_TRY(run_attn_dt(DV_BF16, dh, q, Kc, Vc, B, h, cap, pos, scale, head_idx, head_count, kh_max, at<float>(ws, L.part),
                     at<unsigned>(ws, L.attn_ctr), H, status, st));
  RowsHeads src{head_idx, head_count, H, kh_max, dh, h, WO_s};
  return cuda_status(run_axpy_q8(WOq, d, h * dh, src, bO, out, B, kh_max * dh, 0, status, st));
}

static dv_status check_layer(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p) {
  if (!w || !dims || !p) return DV_ERR_ARG;
  const dv_dims& D = *dims;
  if (!dtype_ok(w->wdtype) || !dtype_ok(w->kvdtype) || !mode_ok(p->mode) || !mode_ok(p->mode_h) || !act_ok(p->act))
    return DV_ERR_ARG;
  if (w->kvdtype != w->wdtype) return DV_ERR_UNSUPPORTED;
  if (!dims_ok(D) || D.h < 1 || D.r < 8 || D.cap < 1) return DV_ERR_ARG;
  if (D.dh != 64 && D.dh != 128) return DV_ERR_UNSUPPORTED;
  if (!w->PA || !w->Wqkv || !w->WOt || !w->Kc || !w->Vc || !w->At || !w->Bm || !w->b1 || !w->W1t || !w->W2t)
    return DV_ERR_ARG;
  if (!ok_ptr(w->PA) || !ok_ptr(w->Wqkv) || !ok_ptr(w->WOt) || !ok_ptr(w->Kc) || !ok_ptr(w->Vc) || !ok_ptr(w->At) ||
      !ok_ptr(w->Bm) || !ok_ptr(w->b1) || !ok_ptr(w->W1t) || !ok_ptr(w->W2t) || !ok_opt(w->bO) || !ok_opt(w->b2) ||
      !ok_opt(w->ln1_g) || !ok_opt(w->ln1_b) || !ok_opt(w->ln2_g) || !ok_opt(w->ln2_b))
    return DV_ERR_ALIGN;
  if (p->k < 0 || p->k_h < 0) return DV_ERR_ARG;
  if (p->exact_kv && D.h > KV_REST_MAX_H) return DV_ERR_UNSUPPORTED;  // the unselected-head list lives in shared memory
  // top-k: the union over B rows has at most min(n, B k) members
  if (p->mode == DV_TOPK && (long long)p->k * D.B > D.k_max && D.N > D.k_max) return DV_ERR_ARG;
  if (p->mode_h == DV_TOPK && (long long)p->k_h * D.B > D.kh_max && D.h > D.kh_max) return DV_ERR_ARG;
  return DV_OK;
}

static dv_status check_layer_call(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p, float* x,
                                  int pos, const dv_layer_io* sel, const dv_layer_io* trace, void* ws,
                                  size_t ws_bytes, Layout* L) {
  DV_CHECK(check_layer(w, dims, p));
  const dv_dims& D = *dims;
  if (!x) return DV_ERR_ARG;
  if (!ok_ptr(x)) return DV_ERR_ALIGN;
  if (pos < 0 || pos >= D.cap) return DV_ERR_ARG;
  if (sel && (!sel->head_idx || !sel->head_count || !sel->idx || !sel->count)) return DV_ERR_ARG;
  if (sel && !ok_opt(sel->yA)) return DV_ERR_ALIGN;
  if (trace && (!ok_opt(trace->yA) || !ok_opt(trace->yM) || !ok_opt(trace->scores) || !ok_opt(trace->scores_h)))
    return DV_ERR_ALIGN;
  *L = layout(D, wbytes_of(w->wdtype));
  return check_ws(*L, ws, ws_bytes);
}

dv_status dv_decode_layer_begin(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p, float* x,
                                int pos, const dv_layer_io* sel, const dv_layer_io* trace, void* ws, size_t ws_bytes,
                                dv_stream_t stream) {
  Layout L;
  DV_CHECK(check_layer_call(w, dims, p, x, pos, sel, trace, ws, ws_bytes, &L));
  return layer_begin(L, ws, w, *dims, p, x, pos, sel, trace, reinterpret_cast<cudaStream_t>(stream));
}

dv_status dv_decode_layer_begin_ahead(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p,
                                      float* x, int pos, const dv_layer_io* sel, const dv_layer_io* trace, void* ws,
                                      size_t ws_bytes, const dv_layer_weights* next, float* next_scores_h,
                                      void* next_ws, size_t next_ws_bytes, dv_stream_t stream) {
  Layout L;
  DV_CHECK(check_layer_call(w, dims, p, x, pos, sel, trace, ws, ws_bytes, &L));
  DV_CHECK(check_layer(next, dims, p));
  if (next->wdtype != w->wdtype) return DV_ERR_UNSUPPORTED;
  if (!next_scores_h || !next_ws) return DV_ERR_ARG;
  if (!ok_ptr(next_scores_h)) return DV_ERR_ALIGN;
  DV_CHECK(check_ws(L, next_ws, next_ws_bytes));
  if (next_ws == ws) return DV_ERR_ARG;
  const Ahead ahead{next, next_scores_h, at<float>(next_ws, L.z)};
  return layer_begin(L, ws, w, *dims, p, x, pos, sel, trace, reinterpret_cast<cudaStream_t>(stream), &ahead);
}

dv_status dv_predict_layer_tail(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p,
                                const dv_layer_io* out, int sets, void* ws, size_t ws_bytes, dv_stream_t stream) {
  DV_CHECK(check_layer(w, dims, p));
  const dv_dims& D = *dims;
  const bool heads = (sets & DV_SET_HEADS) != 0, neurons = (sets & DV_SET_NEURONS) != 0;
  if (!out || sets < 1 || sets > (DV_SET_HEADS | DV_SET_NEURONS)) return DV_ERR_ARG;
  if (heads && (!out->scores_h || !out->head_idx || !out->head_count)) return DV_ERR_ARG;
  if (neurons && (!out->scores || !out->idx || !out->count)) return DV_ERR_ARG;
  if ((heads && !ok_ptr(out->scores_h)) || (neurons && !ok_ptr(out->scores))) return DV_ERR_ALIGN;
  const Layout L = layout(D, wbytes_of(w->wdtype));
  DV_CHECK(check_ws(L, ws, ws_bytes));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (fused_ok(D, w->wdtype)) {
    DV_CHECK(fused_predict_rest(L, ws, w, D, p, heads, neurons, out->scores_h, out->head_idx, out->head_count,
                                out->scores, out->idx, out->count, st));
  } else {
    if (heads)
      DV_TRY(select_any(out->scores_h, D.B, D.h, p->k_h, p->tau_h, p->mode_h, at<uint32_t>(ws, L.bm_h),
                        at<unsigned>(ws, L.sel_ticket_h), out->head_idx, out->head_count, st));
    if (neurons) {
      DV_TRY(predict_scores(L, ws, at<float>(ws, L.z), D.B, D.r, D.N, w->Bm, w->b1, w->wdtype, out->scores, st));
      DV_TRY(select_any(out->scores, D.B, D.N, p->k, p->tau, p->mode, at<uint32_t>(ws, L.bm_m),
                        at<unsigned>(ws, L.sel_ticket_m), out->idx, out->count, st));
    }
  }
  return cuda_status(launch(gate_kernel, dim3(1), dim3(32), 0, st));
}

dv_status dv_decode_layer_end(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p, float* x,
                              int pos, const dv_layer_io* sel, const dv_layer_io* trace, void* ws, size_t ws_bytes,
                              dv_stream_t stream) {
  Layout L;
  DV_CHECK(check_layer_call(w, dims, p, x, pos, sel, trace, ws, ws_bytes, &L));
  return layer_end(L, ws, w, *dims, p, x, pos, sel, trace, reinterpret_cast<cudaStream_t>(stream));
}

dv_status dv_decode_layer_attn(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p, float* x,
                               int pos, const dv_layer_io* sel, const dv_layer_io* trace, void* ws, size_t ws_bytes,
                               dv_stream_t stream) {
  Layout L;
  DV_CHECK(check_layer_call(w, dims, p, x, pos, sel, trace, ws, ws_bytes, &L));
  return layer_attn(L, ws, w, *dims, p, x, pos, sel, trace, reinterpret_cast<cudaStream_t>(stream));
}

dv_status dv_decode_layer_mlp(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p, float* x,
                              const dv_layer_io* sel, const dv_layer_io* trace, void* ws, size_t ws_bytes,
                              dv_stream_t stream) {
  Layout L;
  DV_CHECK(check_layer_call(w, dims, p, x, 0, sel, trace, ws, ws_bytes, &L));
  return layer_mlp(L, ws, w, *dims, p, x, sel, trace, reinterpret_cast<cudaStream_t>(stream));
}

dv_status dv_decode_layer(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p, float* x, int pos,
                          const dv_layer_io* sel, const dv_layer_io* trace, void* ws, size_t ws_bytes,
                          dv_stream_t stream) {
  Layout L;
  DV_CHECK(check_layer_call(w, dims, p, x, pos, sel, trace, ws, ws_bytes, &L));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DV_CHECK(layer_begin(L, ws, w, *dims, p, x, pos, sel, trace, st));
  return layer_end(L, ws, w, *dims, p, x, pos, sel, trace, st);
}

dv_status dv_prefetch_layer(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_io* sel, int pos,
                            int with_w2, dv_stream_t stream) {
  if (!w || !dims || !sel || !sel->head_idx || !sel->head_count || !sel->idx || !sel->count) return DV_ERR_ARG;
  const dv_dims& D = *dims;
  if (!dims_ok(D) || D.h < 1 || pos < 0 || pos >= D.cap) return DV_ERR_ARG;
  if (!dtype_ok(w->wdtype) || !dtype_ok(w->kvdtype)) return DV_ERR_ARG;
  if (!ok_ptr(w->Wqkv) || !ok_ptr(w->WOt) || !ok_ptr(w->Kc) || !ok_ptr(w->Vc) || !ok_ptr(w->W1t) ||
      !ok_ptr(w->W2t))
    return DV_ERR_ALIGN;
  PrefetchArgs a;
  a.Wqkv = static_cast<const char*>(w->Wqkv);
  a.WOt = static_cast<const char*>(w->WOt);
  a.Kc = static_cast<const char*>(w->Kc);
  a.Vc = static_cast<const char*>(w->Vc);
  a.W1t = static_cast<const char*>(w->W1t);
  a.W2t = static_cast<const char*>(w->W2t);
  a.head_idx = sel->head_idx;
  a.head_count = sel->head_count;
  a.idx = sel->idx;
  a.count = sel->count;
  a.kh_max = D.kh_max;
  a.k_max = D.k_max;
  a.B = D.B;
  a.h = D.h;
  a.dh = D.dh;
  a.d = D.d;
  a.N = D.N;
  a.cap = D.cap;
  a.pos = pos;
  a.wbytes = wbytes_of(w->wdtype);
  a.kvbytes = wbytes_of(w->kvdtype);
  a.with_w2 = with_w2 ? 1 : 0;
  return cuda_status(launch(prefetch_layer_kernel, dim3(64), 256, 0, reinterpret_cast<cudaStream_t>(stream), a));
}

dv_status dv_layernorm(const float* x, int B, int d, const float* g, const float* beta, float eps, float* y,
                       dv_stream_t stream) {
  if (!x || !y || B < 1 || B > 16 || d < 8 || d % 8 != 0) return DV_ERR_ARG;
  if (!ok_ptr(x) || !ok_ptr(y) || !ok_opt(g) || !ok_opt(beta)) return DV_ERR_ALIGN;
  return cuda_status(launch(layernorm_kernel, dim3(B), LN_THREADS, 0, reinterpret_cast<cudaStream_t>(stream), x, y, d,
                            g, beta, eps));
}

dv_status dv_predict_layer(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p, const float* y,
                           const dv_layer_io* out, void* ws, size_t ws_bytes, dv_stream_t stream) {
  DV_CHECK(check_layer(w, dims, p));
  const dv_dims& D = *dims;
  if (!y || !out || !out->scores_h || !out->head_idx || !out->head_count || !out->scores || !out->idx || !out->count)
    return DV_ERR_ARG;
  if (!ok_ptr(y) || !ok_ptr(out->scores) || !ok_ptr(out->scores_h)) return DV_ERR_ALIGN;
  const Layout L = layout(D, wbytes_of(w->wdtype));
  DV_CHECK(check_ws(L, ws, ws_bytes));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (fused_ok(D, w->wdtype)) {
    DV_CHECK(fused_predict(L, ws, w, D, p, y, true, true, out->scores_h, out->head_idx, out->head_count, out->scores,
                           out->idx, out->count, st));
  } else {
    DV_CHECK(do_predict_heads(L, ws, y, D.B, D.d, D.h, w->PA, w->wdtype, p->k_h, p->tau_h, p->mode_h, out->scores_h,
                              out->head_idx, out->head_count, st));
    DV_CHECK(do_predict_mlp(L, ws, y, D.B, D.d, D.r, D.N, w->At, w->Bm, w->b1, w->wdtype, p->k, p->tau, p->mode,
                            out->scores, out->idx, out->count, st));
  }
  // consumers on other streams read the sets before their own dependency
  // wait; the gate makes every such consumer start after the sets are done
  return cuda_status(launch(gate_kernel, dim3(1), dim3(32), 0, st));
}

}  // extern "C"

// ===========================================================================
// Selection with file-scope scratch, for callers that cannot allocate
// (dv_topk_static). Layout of the array: the ticket in the first 256 bytes,
// then the per-row selection bitmaps [rows][n/32].
// ===========================================================================

static __device__ __align__(256) unsigned char g_topk_static_scratch[DV_TOPK_STATIC_SCRATCH_BYTES];

namespace {

// Device address of g_topk_static_scratch in the current context, looked up
// on every call: the host-side name is only a stand-in, and after a context
// is torn down and rebuilt (cudaDeviceReset, a host framework resetting the
// device) the module is loaded again and the array may sit elsewhere, so a
// cached address could be stale. The lookup does no allocation.
dv_status static_scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_topk_static_scratch) != cudaSuccess || !p) return DV_ERR_CUDA;
  *out = p;
  return DV_OK;
}

}  // namespace

extern "C" dv_status dv_topk_static(const float* scores, int B, int n, int k, float tau, int mode, int32_t* idx,
                                    int32_t* count, dv_stream_t stream) {
  if (!mode_ok(mode) || !scores || !idx || !count || n < 1 || B < 1) return DV_ERR_ARG;
  if (!ok_ptr(scores)) return DV_ERR_ALIGN;
  if (B > DV_TOPK_STATIC_MAX_ROWS || n > DV_TOPK_STATIC_MAX_N) return DV_ERR_UNSUPPORTED;
  void* base = nullptr;
  DV_CHECK(static_scratch_address(&base));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned* ticket = static_cast<unsigned*>(base);
  uint32_t* bitmaps = reinterpret_cast<uint32_t*>(static_cast<char*>(base) + 256);
  DV_TRY(cudaMemsetAsync(ticket, 0, sizeof(unsigned), st));  // the last-CTA ticket starts at zero
  return cuda_status(select_any(scores, B, n, k, tau, mode, bitmaps, ticket, idx, count, st));
}
