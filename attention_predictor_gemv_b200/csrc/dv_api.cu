// C ABI of the decode library: argument checks, workspace layout, launches.
// Declarations and argument contracts: include/dejavu.h.
#include <atomic>
#include <cstdlib>
#include <map>
#include <cstring>
#include <mutex>

#include "../../include/dejavu.h"
#include "dv_colowner.cuh"

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

// Every kernel asks for the largest shared-memory carveout, so that CTAs of
// different kernels (consecutive ones overlapping under programmatic launch,
// and the two streams of the look-ahead) can share an SM without the SM
// having to drain and reconfigure its L1 / shared split. Cached per kernel.
std::mutex g_carve_mu;
std::map<std::pair<const void*, int>, bool> g_carve_set;

template <typename K>
void prefer_max_shared(K kern) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return;
  const auto key = std::make_pair(reinterpret_cast<const void*>(kern), dev);
  std::lock_guard<std::mutex> lock(g_carve_mu);
  if (g_carve_set.count(key)) return;
  cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  g_carve_set[key] = true;
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
  prefer_max_shared(kern);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Launch as thread-block clusters of `cluster_x` CTAs (plus programmatic
// stream serialisation).
template <typename... KArgs, typename... Args>
cudaError_t launch_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_x,
                           Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  prefer_max_shared(kern);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Raises a kernel's dynamic shared memory limit to `bytes` when needed (the
// default 48 KB covers static plus dynamic). Cached per kernel and device.
std::mutex g_smem_mu;
struct SmemKey {
  const void* fn;
  int dev;
  bool operator<(const SmemKey& o) const { return fn < o.fn || (fn == o.fn && dev < o.dev); }
};
std::map<SmemKey, size_t> g_smem_set;

template <typename K>
cudaError_t allow_smem(K kern, size_t bytes) {
  if (bytes == 0) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const SmemKey key{reinterpret_cast<const void*>(kern), dev};
  std::lock_guard<std::mutex> lock(g_smem_mu);
  auto it = g_smem_set.find(key);
  if (it != g_smem_set.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) g_smem_set[key] = bytes;
  return e;
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
// 0, the selection tickets at 16, 32, 48 and 64, the attention split counters
// [B][kh_max] from 1024, and the neuron-score histograms from 64 KB.
constexpr size_t WS_HEADER = 192 * 1024;
constexpr size_t WS_HIST = 64 * 1024;  // [16][2048] digit histograms of the fused neuron predictor
constexpr int KH_LIMIT = 1000;  // B * kh_max counters must fit the header

// Workspace layout. Offsets in bytes from the workspace base.
struct Layout {
  size_t status, sel_ticket_h, sel_ticket_m, pa_ticket, pb_ticket, attn_ctr, hist, t1;
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
  L.pa_ticket = L.status + 48;
  L.pb_ticket = L.status + 64;
  L.attn_ctr = L.status + 1024;
  L.hist = L.status + WS_HIST;
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
  if (n <= SEL_SMEM_KEYS) {  // keys (top-k) and the union bitmap in shared memory
    const size_t smem = 4ull * n;
    cudaError_t e = allow_smem(select_kernel<true>, smem);
    if (e != cudaSuccess) return e;
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
  cudaError_t e = allow_smem(axpy_rows_kernel<T, NB, Src>, smem);
  if (e != cudaSuccess) return e;
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

// ---------------------------------------------------------------------------
// Fused layer path (dv_fused.cuh)
// ---------------------------------------------------------------------------

constexpr int ATTN_CS = 8;  // CTAs per cluster (per selected head) in attn_out_kernel

int attn_out_S(int pos) { return (pos + 1 + ATTN_CS - 1) / ATTN_CS; }
size_t attn_out_smem(int S, int dh, int kvbytes) { return 2ull * S * dh * kvbytes + 4ull * S; }

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
  const int wb = wbytes_of(wdt), E = 16 / wb;
  if (D.d % (ATTN_CS * E) != 0) return false;
  if ((size_t)D.B * D.d * 4 > 160 * 1024) return false;
  if (attn_out_smem(attn_out_S(D.cap - 1), D.dh, wb) > 190 * 1024) return false;
  if (D.N > SEL_SMEM_KEYS || D.h > HSEL_MAX) return false;
  return true;
}

template <typename K, typename A>
cudaError_t launch_fused(K kern, dim3 grid, size_t smem, cudaStream_t st, const A& a) {
  cudaError_t e = allow_smem(kern, smem);
  if (e != cudaSuccess) return e;
  return launch(kern, grid, FUSED_THREADS, smem, st, a);
}

template <typename T, int NB>
cudaError_t run_attn_in_nb(const AttnInArgs& a, cudaStream_t st) {
  const int rpw = rpw_for(a.d, WT<T>::E);
  const int slots = a.kh_max * 3 * a.dh, per = FUSED_WARPS * rpw;
  const dim3 grid(slots > 0 ? (slots + per - 1) / per : 1);
  const size_t smem = 4ull * a.nb * a.d;
  switch (rpw) {
    case 1: return launch_fused(attn_in_kernel<T, NB, 1, 8>, grid, smem, st, a);
    case 2: return launch_fused(attn_in_kernel<T, NB, 2, 4>, grid, smem, st, a);
    case 4: return launch_fused(attn_in_kernel<T, NB, 4, 2>, grid, smem, st, a);
    default: return launch_fused(attn_in_kernel<T, NB, 8, 1>, grid, smem, st, a);
  }
}

template <typename T>
cudaError_t run_attn_in(const AttnInArgs& a, cudaStream_t st) {
  switch (nb_bucket(a.nb)) {
    case 1: return run_attn_in_nb<T, 1>(a, st);
    case 2: return run_attn_in_nb<T, 2>(a, st);
    case 4: return run_attn_in_nb<T, 4>(a, st);
    case 8: return run_attn_in_nb<T, 8>(a, st);
    default: return run_attn_in_nb<T, 16>(a, st);
  }
}

template <typename KT, int DH, int NB>
cudaError_t run_attn_out_nb(const AttnOutArgs& a, cudaStream_t st) {
  const size_t smem = attn_out_smem(a.S, DH, sizeof(KT));
  auto kern = attn_out_kernel<KT, DH, ATTN_CS, NB>;
  cudaError_t e = allow_smem(kern, smem);
  if (e != cudaSuccess) return e;
  return launch_cluster(kern, dim3(ATTN_CS, a.kh_max > 0 ? a.kh_max : 1), FUSED_THREADS, smem, st, ATTN_CS, a);
}

template <typename KT, int DH>
cudaError_t run_attn_out_dh(const AttnOutArgs& a, cudaStream_t st) {
  switch (nb_bucket(a.nb)) {
    case 1: return run_attn_out_nb<KT, DH, 1>(a, st);
    case 2: return run_attn_out_nb<KT, DH, 2>(a, st);
    case 4: return run_attn_out_nb<KT, DH, 4>(a, st);
    case 8: return run_attn_out_nb<KT, DH, 8>(a, st);
    default: return run_attn_out_nb<KT, DH, 16>(a, st);
  }
}

template <typename KT>
cudaError_t run_attn_out(const AttnOutArgs& a, cudaStream_t st) {
  return a.dh == 64 ? run_attn_out_dh<KT, 64>(a, st) : run_attn_out_dh<KT, 128>(a, st);
}

int mlp_block_grid(int k_max) {
  const int g = (k_max + 7) / 8;
  return g < 1 ? 1 : (g > sm_count() ? sm_count() : g);
}

template <typename T, int NB>
cudaError_t run_mlp_block_nb(const MlpBlockArgs& a, cudaStream_t st) {
  const int rpw = rpw_for(a.d, WT<T>::E);
  const dim3 grid(a.G);
  const size_t smem = 4ull * a.nb * a.d;
  switch (rpw) {
    case 1: return launch_fused(mlp_block_kernel<T, NB, 1, 8>, grid, smem, st, a);
    case 2: return launch_fused(mlp_block_kernel<T, NB, 2, 4>, grid, smem, st, a);
    case 4: return launch_fused(mlp_block_kernel<T, NB, 4, 2>, grid, smem, st, a);
    default: return launch_fused(mlp_block_kernel<T, NB, 8, 1>, grid, smem, st, a);
  }
}

template <typename T>
cudaError_t run_mlp_block(const MlpBlockArgs& a, cudaStream_t st) {
  switch (nb_bucket(a.nb)) {
    case 1: return run_mlp_block_nb<T, 1>(a, st);
    case 2: return run_mlp_block_nb<T, 2>(a, st);
    case 4: return run_mlp_block_nb<T, 4>(a, st);
    case 8: return run_mlp_block_nb<T, 8>(a, st);
    default: return run_mlp_block_nb<T, 16>(a, st);
  }
}

template <typename T, int NB>
cudaError_t run_predict_a_nb(const PredictAArgs& a, cudaStream_t st) {
  const int rows = (a.PA ? a.h : 0) + (a.At ? a.r : 0);
  const int rpw = rpw_for(a.d, WT<T>::E), per = FUSED_WARPS * rpw;
  const dim3 grid(rows > 0 ? (rows + per - 1) / per : 1);
  switch (rpw) {
    case 1: return launch(predict_a_kernel<T, NB, 1, 8>, grid, FUSED_THREADS, 0, st, a);
    case 2: return launch(predict_a_kernel<T, NB, 2, 4>, grid, FUSED_THREADS, 0, st, a);
    case 4: return launch(predict_a_kernel<T, NB, 4, 2>, grid, FUSED_THREADS, 0, st, a);
    default: return launch(predict_a_kernel<T, NB, 8, 1>, grid, FUSED_THREADS, 0, st, a);
  }
}

template <typename T>
cudaError_t run_predict_a(const PredictAArgs& a, cudaStream_t st) {
  switch (nb_bucket(a.nb)) {
    case 1: return run_predict_a_nb<T, 1>(a, st);
    case 2: return run_predict_a_nb<T, 2>(a, st);
    case 4: return run_predict_a_nb<T, 4>(a, st);
    case 8: return run_predict_a_nb<T, 8>(a, st);
    default: return run_predict_a_nb<T, 16>(a, st);
  }
}

template <typename T, int NB>
cudaError_t run_predict_b_nb(const PredictBArgs& a, cudaStream_t st) {
  const int rpw = rpw_for(a.r, WT<T>::E), per = FUSED_WARPS * rpw;
  const dim3 grid((a.N + per - 1) / per);
  switch (rpw) {
    case 1: return launch(predict_b_kernel<T, NB, 1, 8>, grid, FUSED_THREADS, 0, st, a);
    case 2: return launch(predict_b_kernel<T, NB, 2, 4>, grid, FUSED_THREADS, 0, st, a);
    case 4: return launch(predict_b_kernel<T, NB, 4, 2>, grid, FUSED_THREADS, 0, st, a);
    default: return launch(predict_b_kernel<T, NB, 8, 1>, grid, FUSED_THREADS, 0, st, a);
  }
}

template <typename T>
cudaError_t run_predict_b(const PredictBArgs& a, cudaStream_t st) {
  switch (nb_bucket(a.nb)) {
    case 1: return run_predict_b_nb<T, 1>(a, st);
    case 2: return run_predict_b_nb<T, 2>(a, st);
    case 4: return run_predict_b_nb<T, 4>(a, st);
    case 8: return run_predict_b_nb<T, 8>(a, st);
    default: return run_predict_b_nb<T, 16>(a, st);
  }
}

// ---------------------------------------------------------------------------
// Column-owner kernels (dv_colowner.cuh) for batch 1-2
// ---------------------------------------------------------------------------

int co_nv(int d, int E) { return (d + CO_THREADS * E - 1) / (CO_THREADS * E); }
// Rows per group: 8 or more 16-byte loads in flight per thread. The MLP
// kernel also holds the W2 rows and its output slice, so it keeps fewer.
int co_r(int nv) { return nv == 1 ? 8 : nv == 2 ? 4 : nv == 3 ? 3 : 4; }
int co_r_mlp(int nv) { return nv == 1 ? 8 : nv == 2 ? 4 : nv == 3 ? 3 : 2; }
bool co_ok(int nb, int d, int E) { return nb <= 2 && co_nv(d, E) <= 6; }
int co_grid(long long groups) {
  const long long cap = 2ll * sm_count();
  return (int)(groups < 1 ? 1 : (groups > cap ? cap : groups));
}

#define DV_CO_SWITCH(KERN, NB, grid, st, a)                                   \
  switch (nv) {                                                              \
    case 1: return launch(KERN<T, NB, 1, 8>, grid, CO_THREADS, 0, st, a);    \
    case 2: return launch(KERN<T, NB, 2, 4>, grid, CO_THREADS, 0, st, a);    \
    case 3: return launch(KERN<T, NB, 3, 3>, grid, CO_THREADS, 0, st, a);    \
    case 4: return launch(KERN<T, NB, 4, 4>, grid, CO_THREADS, 0, st, a);    \
    case 5: return launch(KERN<T, NB, 5, 4>, grid, CO_THREADS, 0, st, a);    \
    default: return launch(KERN<T, NB, 6, 4>, grid, CO_THREADS, 0, st, a);   \
  }
#define DV_CO_SWITCH_MLP(KERN, NB, grid, st, a)                               \
  switch (nv) {                                                              \
    case 1: return launch(KERN<T, NB, 1, 8>, grid, CO_THREADS, 0, st, a);    \
    case 2: return launch(KERN<T, NB, 2, 4>, grid, CO_THREADS, 0, st, a);    \
    case 3: return launch(KERN<T, NB, 3, 3>, grid, CO_THREADS, 0, st, a);    \
    case 4: return launch(KERN<T, NB, 4, 2>, grid, CO_THREADS, 0, st, a);    \
    case 5: return launch(KERN<T, NB, 5, 2>, grid, CO_THREADS, 0, st, a);    \
    default: return launch(KERN<T, NB, 6, 2>, grid, CO_THREADS, 0, st, a);   \
  }

template <typename T, int NB>
cudaError_t run_attn_in_co_nb(const AttnInArgs& a, cudaStream_t st) {
  const int nv = co_nv(a.d, WT<T>::E), R = co_r(nv);
  const dim3 grid(co_grid(((long long)a.kh_max * 3 * a.dh + R - 1) / R));
  DV_CO_SWITCH(attn_in_co_kernel, NB, grid, st, a)
}

template <typename T, int NB>
cudaError_t run_mlp_block_co_nb(MlpBlockArgs a, cudaStream_t st) {
  const int nv = co_nv(a.d, WT<T>::E), R = co_r_mlp(nv);
  a.G = co_grid(((long long)a.k_max + R - 1) / R);
  const dim3 grid(a.G);
  DV_CO_SWITCH_MLP(mlp_block_co_kernel, NB, grid, st, a)
}

template <typename T, int NB>
cudaError_t run_predict_a_co_nb(const PredictAArgs& a, cudaStream_t st) {
  const int nv = co_nv(a.d, WT<T>::E), R = co_r(nv);
  const int rows = (a.PA ? a.h : 0) + (a.At ? a.r : 0);
  const dim3 grid(co_grid((rows + R - 1) / R));
  DV_CO_SWITCH(predict_a_co_kernel, NB, grid, st, a)
}
#undef DV_CO_SWITCH
#undef DV_CO_SWITCH_MLP

template <typename T>
cudaError_t run_attn_in_any(const AttnInArgs& a, cudaStream_t st) {
  if (co_ok(a.nb, a.d, WT<T>::E))
    return a.nb == 1 ? run_attn_in_co_nb<T, 1>(a, st) : run_attn_in_co_nb<T, 2>(a, st);
  return run_attn_in<T>(a, st);
}

template <typename T>
cudaError_t run_mlp_block_any(const MlpBlockArgs& a, cudaStream_t st) {
  if (co_ok(a.nb, a.d, WT<T>::E))
    return a.nb == 1 ? run_mlp_block_co_nb<T, 1>(a, st) : run_mlp_block_co_nb<T, 2>(a, st);
  return run_mlp_block<T>(a, st);
}

template <typename T>
cudaError_t run_predict_a_any(const PredictAArgs& a, cudaStream_t st) {
  if (co_ok(a.nb, a.d, WT<T>::E))
    return a.nb == 1 ? run_predict_a_co_nb<T, 1>(a, st) : run_predict_a_co_nb<T, 2>(a, st);
  return run_predict_a<T>(a, st);
}

// The head set (heads) and/or the neuron set (neurons) predicted from y:
// predict_a (head scores, z = y A), predict_b (neuron scores + first digit
// histogram), select_finish (exact top-k / threshold of both).
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
  DV_TRY(w->wdtype == DV_BF16 ? run_predict_a_any<bf16>(a, st) : run_predict_a_any<float>(a, st));
  const bool hist_mode = p->mode == DV_TOPK && p->k > 0 && p->k < D.N;
  if (neurons) {
    PredictBArgs b = {};
    b.z = a.z;
    b.Bm = w->Bm;
    b.b1 = w->b1;
    b.N = D.N;
    b.r = D.r;
    b.nb = D.B;
    b.hist_mode = hist_mode ? 1 : 0;
    b.scores = sm;
    b.hist = at<unsigned>(ws, L.hist);
    DV_TRY(w->wdtype == DV_BF16 ? run_predict_b<bf16>(b, st) : run_predict_b<float>(b, st));
  }
  SelectFinishArgs f = {};
  f.scores = sm;
  f.hist = at<unsigned>(ws, L.hist);
  f.bitmaps = at<uint32_t>(ws, L.bm_m);
  f.ticket = at<unsigned>(ws, L.pb_ticket);
  f.neuron_rows = neurons ? D.B : 0;
  f.N = D.N;
  f.nb = D.B;
  f.k = p->k;
  f.mode = p->mode;
  f.tau = p->tau;
  f.idx = midx;
  f.count = mcnt;
  f.scores_h = heads ? sh : nullptr;
  f.h = D.h;
  f.k_h = p->k_h;
  f.mode_h = p->mode_h;
  f.tau_h = p->tau_h;
  f.head_idx = hidx;
  f.head_count = hcnt;
  const int grid = (neurons ? D.B : 0) + (heads ? 1 : 0);
  const size_t smem = 4ull * (neurons && hist_mode ? (D.N > D.h ? D.N : D.h) : D.h);
  DV_TRY(allow_smem(select_finish_kernel, smem));
  DV_TRY(launch(select_finish_kernel, dim3(grid), dim3(SEL_THREADS), smem, st, f));
  return DV_OK;
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
dv_status layer_begin(const Layout& L, void* ws, const dv_layer_weights* w, const dv_dims& D, const dv_layer_params* p,
                      float* x, int pos, const dv_layer_io* sel, const dv_layer_io* trace, cudaStream_t st) {
  const LayerBufs r = layer_bufs(L, ws, sel, trace);
  int* status = at<int>(ws, L.status);
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
    return cuda_status(w->wdtype == DV_BF16 ? run_attn_in_any<bf16>(a, st) : run_attn_in_any<float>(a, st));
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
  if (D.kh_max == 0) return DV_OK;
  float* q = at<float>(ws, L.q);
  return cuda_status(w->wdtype == DV_BF16
                         ? run_qkv<bf16>(w->Wqkv, D.d, D.h, D.dh, yA, D.B, w->bqkv, r.use_hidx, r.use_hcnt, D.kh_max,
                                         q, w->Kc, w->Vc, D.cap, pos, status, st)
                         : run_qkv<float>(w->Wqkv, D.d, D.h, D.dh, yA, D.B, w->bqkv, r.use_hidx, r.use_hcnt,
                                          D.kh_max, q, w->Kc, w->Vc, D.cap, pos, status, st));
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
    return cuda_status(w->kvdtype == DV_BF16 ? run_attn_out<bf16>(b, st) : run_attn_out<float>(b, st));
  }
  if (D.kh_max > 0) {
    float* H = at<float>(ws, L.H);
    const float* q = at<float>(ws, L.q);
    DV_TRY(w->kvdtype == DV_BF16
               ? run_attn<bf16>(D.dh, q, w->Kc, w->Vc, D.B, D.h, D.cap, pos, p->scale, r.use_hidx, r.use_hcnt,
                                D.kh_max, at<float>(ws, L.part), at<unsigned>(ws, L.attn_ctr), H, status, st)
               : run_attn<float>(D.dh, q, w->Kc, w->Vc, D.B, D.h, D.cap, pos, p->scale, r.use_hidx, r.use_hcnt,
                                 D.kh_max, at<float>(ws, L.part), at<unsigned>(ws, L.attn_ctr), H, status, st));
    RowsHeads src{r.use_hidx, r.use_hcnt, H, D.kh_max, D.dh, D.h};
    return cuda_status(w->wdtype == DV_BF16 ? run_axpy<bf16>(w->WOt, D.d, D.h * D.dh, src, w->bO, x, D.B,
                                                             D.kh_max * D.dh, 0, status, st)
                                            : run_axpy<float>(w->WOt, D.d, D.h * D.dh, src, w->bO, x, D.B,
                                                              D.kh_max * D.dh, 0, status, st));
  }
  if (w->bO) {
    RowsHeads none{r.use_hidx, r.use_hcnt, nullptr, 0, D.dh, D.h};
    return cuda_status(w->wdtype == DV_BF16
                           ? run_axpy<bf16>(w->WOt, D.d, D.h * D.dh, none, w->bO, x, D.B, 1, 0, status, st)
                           : run_axpy<float>(w->WOt, D.d, D.h * D.dh, none, w->bO, x, D.B, 1, 0, status, st));
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
    return cuda_status(w->wdtype == DV_BF16 ? run_mlp_block_any<bf16>(c, st) : run_mlp_block_any<float>(c, st));
  }
  DV_TRY(launch(layernorm_kernel, dim3(D.B), LN_THREADS, 0, st, (const float*)x, r.yM, D.d, w->ln2_g, w->ln2_b,
                p->eps));
  if (!sel)
    DV_CHECK(do_predict_mlp(L, ws, r.yM, D.B, D.d, D.r, D.N, w->At, w->Bm, w->b1, w->wdtype, p->k, p->tau, p->mode,
                            r.sm, r.midx, r.mcnt, st));
  return do_sparse_mlp(L, ws, r.yM, D.B, D.d, D.N, w->W1t, w->b1, w->W2t, w->b2, w->wdtype, r.use_midx, r.use_mcnt,
                       D.k_max, x, 1, st);
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
