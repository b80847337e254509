// C ABI of the decode library: argument checks, workspace layout, launches.
// Declarations and argument contracts: include/dejavu.h.
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/dejavu.h"
#include "dv_kernels.cuh"

using namespace dv;
using bf16 = __nv_bfloat16;

namespace {

std::atomic<uint64_t> g_launches{0};

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("DV_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

// Launch with programmatic stream serialisation, so a kernel's launch and
// prologue overlap the tail of the previous kernel on the stream.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

int sm_count() {
  static int n = [] {
    int dev = 0, v = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v > 0 ? v : 148;
  }();
  return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
bool ok_opt(const void* p) { return p == nullptr || aligned16(p); }

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

int nb_bucket(int B) { return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : B <= 8 ? 8 : 16; }

// RPW rows per warp and U column steps so that RPW * U = 8 loads per lane.
int rpw_for(int K, int E) {
  const int vpl = (K / E + 31) / 32;
  return vpl >= 8 ? 1 : vpl >= 4 ? 2 : vpl >= 2 ? 4 : 8;
}

constexpr int ATTN_S_MIN = 32;
// Every layout starts with the same fixed header that holds the counters, so
// calls of different operations may share one workspace: the status word at
// 0, the two selection tickets at 16 and 32, and the attention split counters
// [B][kh_max] from 1024.
constexpr size_t WS_HEADER = 64 * 1024;
constexpr int KH_LIMIT = 1000;  // B * kh_max counters must fit the header

// Workspace layout. Offsets in bytes from the workspace base.
struct Layout {
  size_t status, sel_ticket_h, sel_ticket_m, attn_ctr;
  size_t yA, yM, z, scores_h, bm_h, head_idx, head_count, scores, bm_m, idx, count;
  size_t q, part, H, seg_idx, seg_a, seg_cnt, total;
  int nseg, SEG, nsplit_max;
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
  L.attn_ctr = L.status + 1024;
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

// ---------------------------------------------------------------------------
// Launchers (arguments already checked)
// ---------------------------------------------------------------------------

template <typename T, int NB>
cudaError_t run_dense_gemv_nb(const void* W, int nrows, int K, const float* X, int ldx, int nb, const float* bias,
                              float* out, int ldo, cudaStream_t st) {
  const T* w = static_cast<const T*>(W);
  const int rpw = rpw_for(K, WT<T>::E);
  const int rows_per_cta = GEMV_WARPS * rpw;
  dim3 grid((nrows + rows_per_cta - 1) / rows_per_cta);
  switch (rpw) {
    case 1: return launch(dense_gemv_kernel<T, NB, 1, 8>, grid, GEMV_THREADS, 0, st, w, nrows, K, X, ldx, nb, bias, out, ldo);
    case 2: return launch(dense_gemv_kernel<T, NB, 2, 4>, grid, GEMV_THREADS, 0, st, w, nrows, K, X, ldx, nb, bias, out, ldo);
    case 4: return launch(dense_gemv_kernel<T, NB, 4, 2>, grid, GEMV_THREADS, 0, st, w, nrows, K, X, ldx, nb, bias, out, ldo);
    default: return launch(dense_gemv_kernel<T, NB, 8, 1>, grid, GEMV_THREADS, 0, st, w, nrows, K, X, ldx, nb, bias, out, ldo);
  }
}

template <typename T>
cudaError_t run_dense_gemv(const void* W, int nrows, int K, const float* X, int ldx, int nb, const float* bias,
                           float* out, int ldo, cudaStream_t st) {
  switch (nb_bucket(nb)) {
    case 1: return run_dense_gemv_nb<T, 1>(W, nrows, K, X, ldx, nb, bias, out, ldo, st);
    case 2: return run_dense_gemv_nb<T, 2>(W, nrows, K, X, ldx, nb, bias, out, ldo, st);
    case 4: return run_dense_gemv_nb<T, 4>(W, nrows, K, X, ldx, nb, bias, out, ldo, st);
    case 8: return run_dense_gemv_nb<T, 8>(W, nrows, K, X, ldx, nb, bias, out, ldo, st);
    default: return run_dense_gemv_nb<T, 16>(W, nrows, K, X, ldx, nb, bias, out, ldo, st);
  }
}

cudaError_t run_gemv(dv_dtype dt, const void* W, int nrows, int K, const float* X, int ldx, int nb, const float* bias,
                     float* out, int ldo, cudaStream_t st) {
  return dt == DV_BF16 ? run_dense_gemv<bf16>(W, nrows, K, X, ldx, nb, bias, out, ldo, st)
                       : run_dense_gemv<float>(W, nrows, K, X, ldx, nb, bias, out, ldo, st);
}

cudaError_t run_select(const float* scores, int nrows, int n, int k, float tau, int mode, uint32_t* bm,
                       unsigned* ticket, int32_t* idx, int32_t* count, cudaStream_t st) {
  const bool need_keys = (mode == DV_TOPK) && k > 0 && k < n;
  if (need_keys && n <= SEL_SMEM_KEYS) {
    const size_t smem = 4ull * n;
    static bool attr_set = false;
    if (!attr_set) {
      cudaError_t e = cudaFuncSetAttribute(select_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           4 * SEL_SMEM_KEYS);
      if (e != cudaSuccess) return e;
      attr_set = true;
    }
    return launch(select_kernel<true>, dim3(nrows), SEL_THREADS, smem, st, scores, n, nrows, k, tau, mode, bm, ticket,
                  idx, count);
  }
  return launch(select_kernel<false>, dim3(nrows), SEL_THREADS, 0, st, scores, n, nrows, k, tau, mode, bm, ticket, idx,
                count);
}

template <typename T, int NB>
cudaError_t run_mlp_up_nb(const void* W1t, int d, int N, const float* y, int nb, const float* b1, const int32_t* idx,
                          const int32_t* count, int k_max, int32_t* seg_idx, float* seg_a, int32_t* seg_cnt,
                          int* status, int nseg, cudaStream_t st) {
  const T* w = static_cast<const T*>(W1t);
  dim3 grid(nseg > 0 ? nseg : 1);
  switch (rpw_for(d, WT<T>::E)) {
    case 1: return launch(mlp_up_kernel<T, NB, 1, 8>, grid, GEMV_THREADS, 0, st, w, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status);
    case 2: return launch(mlp_up_kernel<T, NB, 2, 4>, grid, GEMV_THREADS, 0, st, w, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status);
    case 4: return launch(mlp_up_kernel<T, NB, 4, 2>, grid, GEMV_THREADS, 0, st, w, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status);
    default: return launch(mlp_up_kernel<T, NB, 8, 1>, grid, GEMV_THREADS, 0, st, w, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status);
  }
}

template <typename T, int NB, class Src>
cudaError_t run_axpy_st(const void* W, int d, int nrows_w, Src src, const float* bias, float* out, int nb, int k_max,
                        size_t smem, int* status, cudaStream_t st) {
  constexpr int E = WT<T>::E;
  const int tiles = (d + AX_THREADS * E - 1) / (AX_THREADS * E);
  int G = (2 * sm_count() + tiles - 1) / tiles;
  const int gmax = (k_max + 3) / 4;
  if (G > gmax) G = gmax;
  if (G < 1) G = 1;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(axpy_rows_kernel<T, NB, Src>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch(axpy_rows_kernel<T, NB, Src>, dim3(tiles, G), AX_THREADS, smem, st, static_cast<const T*>(W), d,
                nrows_w, src, bias, out, nb, G, status);
}

template <typename T, class Src>
cudaError_t run_axpy(const void* W, int d, int nrows_w, Src src, const float* bias, float* out, int nb, int k_max,
                     size_t smem, int* status, cudaStream_t st) {
  switch (nb_bucket(nb)) {
    case 1: return run_axpy_st<T, 1>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
    case 2: return run_axpy_st<T, 2>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
    case 4: return run_axpy_st<T, 4>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
    case 8: return run_axpy_st<T, 8>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
    default: return run_axpy_st<T, 16>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
  }
}

template <typename T>
cudaError_t run_mlp_up(const void* W1t, int d, int N, const float* y, int nb, const float* b1, const int32_t* idx,
                       const int32_t* count, int k_max, int32_t* seg_idx, float* seg_a, int32_t* seg_cnt, int* status,
                       int nseg, cudaStream_t st) {
  switch (nb_bucket(nb)) {
    case 1: return run_mlp_up_nb<T, 1>(W1t, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, nseg, st);
    case 2: return run_mlp_up_nb<T, 2>(W1t, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, nseg, st);
    case 4: return run_mlp_up_nb<T, 4>(W1t, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, nseg, st);
    case 8: return run_mlp_up_nb<T, 8>(W1t, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, nseg, st);
    default: return run_mlp_up_nb<T, 16>(W1t, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, nseg, st);
  }
}

template <typename T, int NB>
cudaError_t run_qkv_nb(const void* Wqkv, int d, int h, int dh, const float* y, int nb, const float* bqkv,
                       const int32_t* head_idx, const int32_t* head_count, int kh_max, float* q, void* Kc, void* Vc,
                       int cap, int pos, int* status, cudaStream_t st) {
  const T* w = static_cast<const T*>(Wqkv);
  const int rpw = rpw_for(d, WT<T>::E);
  const int slots = kh_max * 3 * dh;
  const int per_cta = GEMV_WARPS * rpw;
  dim3 grid((slots + per_cta - 1) / per_cta > 0 ? (slots + per_cta - 1) / per_cta : 1);
  T* K = static_cast<T*>(Kc);
  T* V = static_cast<T*>(Vc);
  switch (rpw) {
    case 1: return launch(qkv_kernel<T, NB, 1, 8>, grid, GEMV_THREADS, 0, st, w, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, K, V, cap, pos, status);
    case 2: return launch(qkv_kernel<T, NB, 2, 4>, grid, GEMV_THREADS, 0, st, w, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, K, V, cap, pos, status);
    case 4: return launch(qkv_kernel<T, NB, 4, 2>, grid, GEMV_THREADS, 0, st, w, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, K, V, cap, pos, status);
    default: return launch(qkv_kernel<T, NB, 8, 1>, grid, GEMV_THREADS, 0, st, w, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, K, V, cap, pos, status);
  }
}

template <typename T>
cudaError_t run_qkv(const void* Wqkv, int d, int h, int dh, const float* y, int nb, const float* bqkv,
                    const int32_t* head_idx, const int32_t* head_count, int kh_max, float* q, void* Kc, void* Vc,
                    int cap, int pos, int* status, cudaStream_t st) {
  switch (nb_bucket(nb)) {
    case 1: return run_qkv_nb<T, 1>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos, status, st);
    case 2: return run_qkv_nb<T, 2>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos, status, st);
    case 4: return run_qkv_nb<T, 4>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos, status, st);
    case 8: return run_qkv_nb<T, 8>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos, status, st);
    default: return run_qkv_nb<T, 16>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos, status, st);
  }
}

// Keys per split: the largest of 64 / 32 that still gives >= 2 CTAs per SM.
int attn_split_len(int B, int kh_max, int pos) {
  const int want = 2 * sm_count();
  if ((long long)B * kh_max * ((pos + 1 + 63) / 64) >= want) return 64;
  return 32;
}

template <typename KT, int DH>
cudaError_t run_attn_dh(const float* q, const void* Kc, const void* Vc, int B, int h, int cap, int pos, float scale,
                        const int32_t* head_idx, const int32_t* head_count, int kh_max, float* part, unsigned* ctr,
                        float* H, int* status, cudaStream_t st) {
  const int S = (sizeof(KT) * DH * 64 * 2 <= 32768) ? attn_split_len(B, kh_max, pos) : 32;
  const int nsplit = (pos + 1 + S - 1) / S;
  dim3 grid(nsplit, kh_max, B);
  const KT* K = static_cast<const KT*>(Kc);
  const KT* V = static_cast<const KT*>(Vc);
  if constexpr (sizeof(KT) * DH * 64 * 2 <= 32768) {  // K and V tiles in static shared memory
    if (S == 64)
      return launch(attn_split_kernel<KT, DH, 64>, grid, ATTN_THREADS, 0, st, q, K, V, h, cap, pos, scale, head_idx,
                    head_count, kh_max, nsplit, part, ctr, H, status);
  }
  return launch(attn_split_kernel<KT, DH, 32>, grid, ATTN_THREADS, 0, st, q, K, V, h, cap, pos, scale, head_idx,
                head_count, kh_max, nsplit, part, ctr, H, status);
}

template <typename KT>
cudaError_t run_attn(int dh, const float* q, const void* Kc, const void* Vc, int B, int h, int cap, int pos,
                     float scale, const int32_t* head_idx, const int32_t* head_count, int kh_max, float* part,
                     unsigned* ctr, float* H, int* status, cudaStream_t st) {
  if (dh == 64)
    return run_attn_dh<KT, 64>(q, Kc, Vc, B, h, cap, pos, scale, head_idx, head_count, kh_max, part, ctr, H, status, st);
  return run_attn_dh<KT, 128>(q, Kc, Vc, B, h, cap, pos, scale, head_idx, head_count, kh_max, part, ctr, H, status, st);
}

// ---------------------------------------------------------------------------
// Operation bodies shared by the public entry points
// ---------------------------------------------------------------------------

dv_status do_predict_mlp(const Layout& L, void* ws, const float* y, int B, int d, int r, int N, const void* At,
                         const void* Bm, const float* b1, dv_dtype dt, int k, float tau, int mode, float* scores,
                         int32_t* idx, int32_t* count, cudaStream_t st) {
  float* z = at<float>(ws, L.z);
  DV_TRY(run_gemv(dt, At, r, d, y, d, B, nullptr, z, r, st));
  DV_TRY(run_gemv(dt, Bm, N, r, z, r, B, b1, scores, N, st));
  DV_TRY(run_select(scores, B, N, k, tau, mode, at<uint32_t>(ws, L.bm_m), at<unsigned>(ws, L.sel_ticket_m), idx, count,
                    st));
  return DV_OK;
}

dv_status do_predict_heads(const Layout& L, void* ws, const float* y, int B, int d, int h, const void* PA, dv_dtype dt,
                           int k_h, float tau, int mode, float* scores, int32_t* head_idx, int32_t* head_count,
                           cudaStream_t st) {
  DV_TRY(run_gemv(dt, PA, h, d, y, d, B, nullptr, scores, h, st));
  DV_TRY(run_select(scores, B, h, k_h, tau, mode, at<uint32_t>(ws, L.bm_h), at<unsigned>(ws, L.sel_ticket_h), head_idx,
                    head_count, st));
  return DV_OK;
}

dv_status do_sparse_mlp(const Layout& L, void* ws, const float* y, int B, int d, int N, const void* W1t,
                        const float* b1, const void* W2t, const float* b2, dv_dtype dt, const int32_t* idx,
                        const int32_t* count, int k_max, float* out, int accumulate, cudaStream_t st) {
  if (!accumulate) DV_TRY(cudaMemsetAsync(out, 0, 4ull * B * d, st));
  int* status = at<int>(ws, L.status);
  int32_t* seg_idx = at<int32_t>(ws, L.seg_idx);
  float* seg_a = at<float>(ws, L.seg_a);
  int32_t* seg_cnt = at<int32_t>(ws, L.seg_cnt);
  if (L.nseg == 0) {
    if (b2) {  // nothing selected: out (+)= b2 only
      RowsHeads none{idx, count, nullptr, 0, 1, 0};
      return cuda_status(dt == DV_BF16 ? run_axpy<bf16>(W2t, d, N, none, b2, out, B, 1, 0, status, st)
                                       : run_axpy<float>(W2t, d, N, none, b2, out, B, 1, 0, status, st));
    }
    return DV_OK;
  }
  if (dt == DV_BF16)
    DV_TRY(run_mlp_up<bf16>(W1t, d, N, y, B, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, L.nseg, st));
  else
    DV_TRY(run_mlp_up<float>(W1t, d, N, y, B, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, L.nseg, st));
  RowsMlp src{seg_idx, seg_a, seg_cnt, L.nseg, L.SEG};
  const size_t smem = 4ull * (L.nseg + 1);
  return cuda_status(dt == DV_BF16 ? run_axpy<bf16>(W2t, d, N, src, b2, out, B, k_max, smem, status, st)
                                   : run_axpy<float>(W2t, d, N, src, b2, out, B, k_max, smem, status, st));
}

dv_status do_sparse_mha(const Layout& L, void* ws, const float* y, int B, int d, int h, int dh, const void* Wqkv,
                        const float* bqkv, const void* WOt, const float* bO, dv_dtype dt, void* Kc, void* Vc, int cap,
                        int pos, float scale, const int32_t* head_idx, const int32_t* head_count, int kh_max,
                        float* out, int accumulate, cudaStream_t st) {
  if (!accumulate) DV_TRY(cudaMemsetAsync(out, 0, 4ull * B * d, st));
  int* status = at<int>(ws, L.status);
  if (kh_max == 0) {
    if (bO) {
      RowsHeads none{head_idx, head_count, nullptr, 0, dh, h};
      return cuda_status(dt == DV_BF16 ? run_axpy<bf16>(WOt, d, h * dh, none, bO, out, B, 1, 0, status, st)
                                       : run_axpy<float>(WOt, d, h * dh, none, bO, out, B, 1, 0, status, st));
    }
    return DV_OK;
  }
  float* q = at<float>(ws, L.q);
  float* H = at<float>(ws, L.H);
  if (dt == DV_BF16) {
    DV_TRY(run_qkv<bf16>(Wqkv, d, h, dh, y, B, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos, status, st));
    DV_TRY(run_attn<bf16>(dh, q, Kc, Vc, B, h, cap, pos, scale, head_idx, head_count, kh_max, at<float>(ws, L.part),
                          at<unsigned>(ws, L.attn_ctr), H, status, st));
  } else {
    DV_TRY(run_qkv<float>(Wqkv, d, h, dh, y, B, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos, status, st));
    DV_TRY(run_attn<float>(dh, q, Kc, Vc, B, h, cap, pos, scale, head_idx, head_count, kh_max, at<float>(ws, L.part),
                           at<unsigned>(ws, L.attn_ctr), H, status, st));
  }
  RowsHeads src{head_idx, head_count, H, kh_max, dh, h};
  return cuda_status(dt == DV_BF16 ? run_axpy<bf16>(WOt, d, h * dh, src, bO, out, B, kh_max * dh, 0, status, st)
                                   : run_axpy<float>(WOt, d, h * dh, src, bO, out, B, kh_max * dh, 0, status, st));
}

int wbytes_of(dv_dtype t) { return t == DV_BF16 ? 2 : 4; }
bool dtype_ok(int t) { return t == DV_F32 || t == DV_BF16; }
bool mode_ok(int m) { return m == DV_TOPK || m == DV_THRESHOLD; }

dv_status check_ws(const Layout& L, void* ws, size_t ws_bytes) {
  if (!ok_ptr(ws)) return ws ? DV_ERR_ALIGN : DV_ERR_ARG;
  if (ws_bytes < L.total) return DV_ERR_WORKSPACE;
  return DV_OK;
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
  return layout(D, 2).total > layout(D, 4).total ? layout(D, 2).total : layout(D, 4).total;
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
  return cuda_status(run_select(scores, B, n, k, tau, mode, at<uint32_t>(ws, L.bm_m), at<unsigned>(ws, L.sel_ticket_m),
                                idx, count, reinterpret_cast<cudaStream_t>(stream)));
}

dv_status dv_sparse_mlp(const float* y, int B, int d, int N, const void* W1t, const float* b1, const void* W2t,
                        const float* b2, dv_dtype wdtype, const int32_t* idx, const int32_t* count, int k_max,
                        float* out, int accumulate, void* ws, size_t ws_bytes, dv_stream_t stream) {
  if (!dtype_ok(wdtype)) return DV_ERR_ARG;
  if (!y || !W1t || !b1 || !W2t || !idx || !count || !out) return DV_ERR_ARG;
  if (!ok_ptr(y) || !ok_ptr(W1t) || !ok_ptr(W2t) || !ok_ptr(out) || !ok_opt(b2)) return DV_ERR_ALIGN;
  dv_dims D = {B, d, N, 0, 0, 0, 0, k_max, 0};
  if (!dims_ok(D)) return DV_ERR_ARG;
  const Layout L = layout(D, wbytes_of(wdtype));
  DV_CHECK(check_ws(L, ws, ws_bytes));
  return do_sparse_mlp(L, ws, y, B, d, N, W1t, b1, W2t, b2, wdtype, idx, count, k_max, out, accumulate,
                       reinterpret_cast<cudaStream_t>(stream));
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

static dv_status check_layer(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p) {
  if (!w || !dims || !p) return DV_ERR_ARG;
  const dv_dims& D = *dims;
  if (!dtype_ok(w->wdtype) || !dtype_ok(w->kvdtype) || !mode_ok(p->mode) || !mode_ok(p->mode_h)) return DV_ERR_ARG;
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
  // top-k: the union over B rows has at most min(n, B k) members
  if (p->mode == DV_TOPK && (long long)p->k * D.B > D.k_max && D.N > D.k_max) return DV_ERR_ARG;
  if (p->mode_h == DV_TOPK && (long long)p->k_h * D.B > D.kh_max && D.h > D.kh_max) return DV_ERR_ARG;
  return DV_OK;
}

dv_status dv_decode_layer(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p, float* x, int pos,
                          const dv_layer_io* sel, const dv_layer_io* trace, void* ws, size_t ws_bytes,
                          dv_stream_t stream) {
  DV_CHECK(check_layer(w, dims, p));
  const dv_dims& D = *dims;
  if (!x) return DV_ERR_ARG;
  if (!ok_ptr(x)) return DV_ERR_ALIGN;
  if (pos < 0 || pos >= D.cap) return DV_ERR_ARG;
  if (sel && (!sel->head_idx || !sel->head_count || !sel->idx || !sel->count)) return DV_ERR_ARG;
  const Layout L = layout(D, wbytes_of(w->wdtype));
  DV_CHECK(check_ws(L, ws, ws_bytes));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const dv_layer_io none = {};
  const dv_layer_io& t = trace ? *trace : none;
  float* yA = t.yA ? t.yA : at<float>(ws, L.yA);
  float* yM = t.yM ? t.yM : at<float>(ws, L.yM);
  if (!ok_ptr(yA) || !ok_ptr(yM)) return DV_ERR_ALIGN;
  float* sh = t.scores_h ? t.scores_h : at<float>(ws, L.scores_h);
  int32_t* hidx = t.head_idx ? t.head_idx : at<int32_t>(ws, L.head_idx);
  int32_t* hcnt = t.head_count ? t.head_count : at<int32_t>(ws, L.head_count);
  float* sm = t.scores ? t.scores : at<float>(ws, L.scores);
  int32_t* midx = t.idx ? t.idx : at<int32_t>(ws, L.idx);
  int32_t* mcnt = t.count ? t.count : at<int32_t>(ws, L.count);
  const int32_t* use_hidx = sel ? sel->head_idx : hidx;
  const int32_t* use_hcnt = sel ? sel->head_count : hcnt;
  const int32_t* use_midx = sel ? sel->idx : midx;
  const int32_t* use_mcnt = sel ? sel->count : mcnt;

  if (sel && sel->yA) {
    if (!ok_ptr(sel->yA)) return DV_ERR_ALIGN;
    yA = sel->yA;  // LN1(x) computed by the caller
  } else {
    DV_TRY(launch(layernorm_kernel, dim3(D.B), LN_THREADS, 0, st, (const float*)x, yA, D.d, w->ln1_g, w->ln1_b,
                  p->eps));
  }
  if (!sel)
    DV_CHECK(do_predict_heads(L, ws, yA, D.B, D.d, D.h, w->PA, w->wdtype, p->k_h, p->tau_h, p->mode_h, sh, hidx, hcnt,
                              st));
  DV_CHECK(do_sparse_mha(L, ws, yA, D.B, D.d, D.h, D.dh, w->Wqkv, w->bqkv, w->WOt, w->bO, w->wdtype, w->Kc, w->Vc,
                         D.cap, pos, p->scale, use_hidx, use_hcnt, D.kh_max, x, 1, st));
  DV_TRY(launch(layernorm_kernel, dim3(D.B), LN_THREADS, 0, st, (const float*)x, yM, D.d, w->ln2_g, w->ln2_b, p->eps));
  if (!sel)
    DV_CHECK(do_predict_mlp(L, ws, yM, D.B, D.d, D.r, D.N, w->At, w->Bm, w->b1, w->wdtype, p->k, p->tau, p->mode, sm,
                            midx, mcnt, st));
  DV_CHECK(do_sparse_mlp(L, ws, yM, D.B, D.d, D.N, w->W1t, w->b1, w->W2t, w->b2, w->wdtype, use_midx, use_mcnt,
                         D.k_max, x, 1, st));
  return DV_OK;
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
  DV_CHECK(do_predict_heads(L, ws, y, D.B, D.d, D.h, w->PA, w->wdtype, p->k_h, p->tau_h, p->mode_h, out->scores_h,
                            out->head_idx, out->head_count, st));
  DV_CHECK(do_predict_mlp(L, ws, y, D.B, D.d, D.r, D.N, w->At, w->Bm, w->b1, w->wdtype, p->k, p->tau, p->mode,
                          out->scores, out->idx, out->count, st));
  return DV_OK;
}

}  // extern "C"

// ===========================================================================
// Selection with file-scope scratch, for callers that cannot allocate
// (dv_topk_static). Layout of the array: the ticket in the first 256 bytes,
// then the per-row selection bitmaps [rows][n/32].
// ===========================================================================

static __device__ __align__(256) unsigned char g_topk_static_scratch[DV_TOPK_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_addr[kMaxDevices] = {};

// Device address of g_topk_static_scratch on the current device, looked up
// once per device (the host-side name is only a stand-in for it).
dv_status static_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return DV_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_topk_static_scratch) != cudaSuccess || !p) return DV_ERR_CUDA;
    g_static_addr[dev] = p;
  }
  *out = g_static_addr[dev];
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
  return cuda_status(run_select(scores, B, n, k, tau, mode, bitmaps, ticket, idx, count, st));
}
