// dsa_api.cu — the extern "C" entry points declared in include/dsa_index.h.
//
// Host side only: argument validation, workspace layout, TMA tensor-map
// encoding and kernel dispatch.  Nothing here allocates device memory or
// synchronises a stream (except dsa_check_status, whose job that is).
#include <cstdio>
#include <cstring>
#include <mutex>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

int current_device(int* dev_out, int* sms_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
  static int sms_cache[64];
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= 64) return DSA_ERR_DEVICE;
  if (sms_cache[dev] == 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return DSA_ERR_CUDA;
    if (major != 10 || minor != 0 || sms < 1) return DSA_ERR_DEVICE;  // only sm_100a code is built
    sms_cache[dev] = sms;
  }
  if (dev_out) *dev_out = dev;
  if (sms_out) *sms_out = sms_cache[dev];
  return DSA_OK;
}

void* driver_entry(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return p;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// 2-D bf16 tensor map over [rows, inner] with a box of 64 elements (128 B)
// x box_rows rows, 128-byte swizzle (the layout the MMA descriptors expect).
int make_map_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t inner, uint32_t box_rows) {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] { fn = reinterpret_cast<EncodeTiledFn>(driver_entry("cuTensorMapEncodeTiled")); });
  if (!fn) return DSA_ERR_CUDA;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa

using namespace dsa;

namespace {

constexpr int kMaxK = 65536;

struct DeviceInfo {
  int sms = 0;
};

int device_info(DeviceInfo& out) { return current_device(nullptr, &out.sms); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elt_size(int dt) { return dt == DSA_DTYPE_FP32 ? 4 : (dt == DSA_DTYPE_BF16 ? 2 : 1); }

// Simple bump layout over the caller's workspace (256-byte aligned pieces).
struct Layout {
  size_t off = sizeof(WsHeader);
  size_t take(size_t bytes) {
    size_t o = off;
    off += (bytes + 255) & ~size_t(255);
    return o;
  }
};

// bf16 queries with bf16 or fp8 keys at H = 64, d = 128 run on the tensor
// cores; fp8 keys are first widened to bf16 (exactly) in the workspace and
// their per-key scale is applied to the score in the epilogue.
bool use_tc(int H, int d, int q_dtype, int k_dtype) {
  return q_dtype == DSA_DTYPE_BF16 && (k_dtype == DSA_DTYPE_BF16 || k_dtype == DSA_DTYPE_FP8_E4M3) && H == 64 &&
         d == 128;
}

bool needs_widen(int H, int d, int q_dtype, int k_dtype) {
  return use_tc(H, d, q_dtype, k_dtype) && k_dtype == DSA_DTYPE_FP8_E4M3;
}

int check_common(int H, int d, int k, int q_dtype, int k_dtype) {
  if (H < 1 || H > 128 || d < 1 || d > 256 || H * d > 8192) return DSA_ERR_UNSUPPORTED;
  if (k < 1 || k > kMaxK) return DSA_ERR_INVALID_ARG;
  if (q_dtype != DSA_DTYPE_BF16 && q_dtype != DSA_DTYPE_FP32) return DSA_ERR_UNSUPPORTED;
  if (k_dtype != DSA_DTYPE_BF16 && k_dtype != DSA_DTYPE_FP32 && k_dtype != DSA_DTYPE_FP8_E4M3)
    return DSA_ERR_UNSUPPORTED;
  if (q_dtype == DSA_DTYPE_FP32 && k_dtype == DSA_DTYPE_BF16) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

int simt_grid(const DeviceInfo& di, int64_t tasks) {
  int64_t g = (tasks + 1) / 2;
  const int64_t cap = (int64_t)di.sms * 4;
  return (int)(g < cap ? (g < 1 ? 1 : g) : cap);
}

// Offset of the widened (bf16) copy of fp8 keys, taken first in every plan.
size_t take_widen(Layout& L, int64_t n_keys, int H, int d, int q_dtype, int k_dtype) {
  return needs_widen(H, d, q_dtype, k_dtype) ? L.take((size_t)n_keys * d * 2) : 0;
}

int widen_keys(const void* K, int64_t n_keys, int d, uint8_t* ws, size_t off, cudaStream_t st) {
  return launch_e4m3_to_bf16(static_cast<const uint8_t*>(K), n_keys * d, ws + off, st);
}

// Dense / proxy-scan workspace pieces.
struct DensePlan {
  bool tc;
  int grid;
  int64_t cand_cap;
  size_t cand_off;
  size_t total;
};

DensePlan plan_dense(const DeviceInfo& di, int T, int N, int H, int d, int q_dtype, int k_dtype, Layout& L) {
  DensePlan p;
  p.tc = use_tc(H, d, q_dtype, k_dtype);
  // candidate lists: a multiple of 4 tiles of 128 keys, so that a team of
  // 1, 2 or 4 warpgroups splits them into equal per-warp segments that each
  // hold every key of the tiles that warp owns
  p.cand_cap = ((int64_t)N + 511) / 512 * 512;
  if (p.tc) {
    const int units = (T + 3) / 4;
    p.grid = units < di.sms ? units : di.sms;
    p.cand_off = L.take((size_t)p.grid * 4 * p.cand_cap * sizeof(uint2));
  } else {
    p.grid = simt_grid(di, T);
    p.cand_off = L.take((size_t)p.grid * 2 * p.cand_cap * sizeof(uint2));
  }
  p.total = L.off;
  return p;
}

// K / k_dtype: for the tensor-core path the keys as bf16 (fp8 keys already
// widened) with K_scale their per-key scale or null.
int run_dense_rows(const DeviceInfo& di, const DensePlan& p, const void* Q, const float* w, const void* K,
                   const float* K_scale, int n_rows, int N, int H, int d, int64_t pos_base, int64_t pos_mul,
                   int64_t pos_add, int64_t pos_clamp, int k, int q_dtype, int k_dtype, int32_t* idx, float* val,
                   uint8_t* ws, float* dbg, int64_t dbg_ld, cudaStream_t st, int pos_shift = 0) {
  int* status = reinterpret_cast<int*>(ws);
  uint2* cand = reinterpret_cast<uint2*>(ws + p.cand_off);
  if (p.tc) {
    CUtensorMap tmQ, tmK;
    int r = make_map_bf16(&tmQ, Q, (uint64_t)n_rows * H, (uint64_t)d, 64);
    if (r != DSA_OK) return r;
    r = make_map_bf16(&tmK, K, (uint64_t)N, (uint64_t)d, 128);
    if (r != DSA_OK) return r;
    TcArgs a;
    memset(&a, 0, sizeof(a));
    a.kind = 0;
    a.k_scale = K_scale;
    a.n_rows = n_rows;
    a.n_units = (n_rows + 3) / 4;
    a.k = k;
    a.pos_base = pos_base;
    a.pos_mul = pos_mul;
    a.pos_add = pos_add;
    a.pos_clamp = pos_clamp;
    a.pos_shift = pos_shift;
    a.w = w;
    a.out_idx = idx;
    a.out_val = val;
    a.out_ld = k;
    a.cand = cand;
    a.cand_cap = p.cand_cap;
    a.status = status;
    a.dbg_scores = dbg;
    a.dbg_ld = dbg_ld;
    const int grid = a.n_units < p.grid ? a.n_units : p.grid;
    return launch_tc_index(tmQ, tmK, a, grid, st);
  }
  if (pos_mul != 1 || pos_add != 0) return DSA_ERR_UNSUPPORTED;  // proxy rows use the tensor-core kernel
  SimtArgs a;
  memset(&a, 0, sizeof(a));
  a.kind = 0;
  a.n_tasks = n_rows;
  a.H = H;
  a.d = d;
  a.k = k;
  a.q_dtype = q_dtype;
  a.k_dtype = k_dtype;
  a.Q = Q;
  a.w = w;
  a.K = K;
  a.K_scale = K_scale;
  a.q_pos0 = pos_base;
  a.out_idx = idx;
  a.out_val = val;
  a.out_ld = k;
  a.cand = cand;
  a.cand_cap = p.cand_cap;
  a.status = status;
  a.dbg_scores = dbg;
  a.dbg_ld = dbg_ld;
  const int grid = simt_grid(di, n_rows) < p.grid ? simt_grid(di, n_rows) : p.grid;
  return launch_simt_index(a, grid, st);
}

// Empty calls: no query rows (prefill T = 0, decode B = 0).  Nothing is
// computed and nothing is launched; the shape arguments are still checked
// and the workspace needs only its status word.
constexpr size_t kEmptyWorkspaceBytes = 256;

int empty_workspace(size_t* bytes) {
  *bytes = kEmptyWorkspaceBytes;
  return DSA_OK;
}

int empty_prefill(int N, int H, int d, int k, int q_dtype, int k_dtype, int64_t q_pos0) {
  const int r = check_common(H, d, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  return (N < 0 || q_pos0 < 0 || q_pos0 > (int64_t)N) ? DSA_ERR_INVALID_ARG : DSA_OK;
}

int empty_decode(int total_q, int64_t total_keys, int H, int d, int k, int q_dtype, int k_dtype) {
  const int r = check_common(H, d, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  return (total_q != 0 || total_keys != 0) ? DSA_ERR_INVALID_ARG : DSA_OK;
}

bool group_args_ok(int k, int group, int bank, int mode) {
  return group >= 1 && bank >= k && bank <= kMaxBank &&
         (mode == DSA_GROUP_REFINE || mode == DSA_GROUP_REUSE || mode == DSA_GROUP_REFINE_LOCAL);
}

int validate_dense(const void* Q, const float* w, const void* K, const float* K_scale, int T, int N, int H, int d,
                   int64_t q_pos0, int k, int q_dtype, int k_dtype) {
  int r = check_common(H, d, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (!Q || !w || !K) return DSA_ERR_INVALID_ARG;
  if (T < 1 || N < 1 || q_pos0 < 0 || q_pos0 + (int64_t)T > (int64_t)N) return DSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(w)) return DSA_ERR_INVALID_ARG;
  if ((k_dtype == DSA_DTYPE_FP8_E4M3) != (K_scale != nullptr)) return DSA_ERR_INVALID_ARG;
  if ((int64_t)T * H * d >= ((int64_t)1 << 40)) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

}  // namespace

extern "C" {

const char* dsa_status_string(int status) {
  switch (status) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case DSA_ERR_WORKSPACE: return "workspace too small";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "device-side wait timed out";
    case DSA_ERR_DEVICE: return "device is not sm_100";
    case DSA_ERR_INTERNAL: return "device-side consistency check failed";
    default: return "unknown status";
  }
}

int dsa_version(void) { return 100; }

int dsa_debug_set_wait(unsigned int budget_us, int hold_first_tile) {
  set_wait_controls(budget_us, hold_first_tile);
  return DSA_OK;
}

int dsa_check_status(void* workspace, void* stream) {
  if (!workspace) return DSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  int h[2] = {0, 0};
  if (cudaMemcpy(h, workspace, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return DSA_ERR_CUDA;
  if (h[0] != 0) {
    const int z[2] = {0, 0};
    if (cudaMemcpy(workspace, z, sizeof(z), cudaMemcpyHostToDevice) != cudaSuccess) return DSA_ERR_CUDA;
    return h[0];
  }
  return DSA_OK;
}

int dsa_index_dense_workspace_size(int T, int N, int H, int d, int k, int q_dtype, int k_dtype, size_t* bytes) {
  if (!bytes) return DSA_ERR_INVALID_ARG;
  int r = check_common(H, d, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (T < 0 || N < 0) return DSA_ERR_INVALID_ARG;
  if (T == 0) return empty_workspace(bytes);
  if (N < 1) return DSA_ERR_INVALID_ARG;
  DeviceInfo di;
  if ((r = device_info(di)) != DSA_OK) return r;
  Layout L;
  take_widen(L, N, H, d, q_dtype, k_dtype);
  *bytes = plan_dense(di, T, N, H, d, q_dtype, k_dtype, L).total;
  return DSA_OK;
}

int dsa_index_dense(const void* Q, const float* w, const void* K, const float* K_scale, int T, int N, int H, int d,
                    int64_t q_pos0, int k, int q_dtype, int k_dtype, int32_t* idx, float* val, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (T == 0) return empty_prefill(N, H, d, k, q_dtype, k_dtype, q_pos0);
  int r = validate_dense(Q, w, K, K_scale, T, N, H, d, q_pos0, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (!idx || !val || !workspace) return DSA_ERR_INVALID_ARG;
  DeviceInfo di;
  if ((r = device_info(di)) != DSA_OK) return r;
  Layout L;
  const size_t wo = take_widen(L, N, H, d, q_dtype, k_dtype);
  DensePlan p = plan_dense(di, T, N, H, d, q_dtype, k_dtype, L);
  if (workspace_bytes < p.total) return DSA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (needs_widen(H, d, q_dtype, k_dtype)) {
    if ((r = widen_keys(K, N, d, ws, wo, st)) != DSA_OK) return r;
    return run_dense_rows(di, p, Q, w, ws + wo, K_scale, T, N, H, d, q_pos0, 1, 0, (int64_t)T - 1, k, q_dtype,
                          DSA_DTYPE_BF16, idx, val, ws, nullptr, 0, st);
  }
  return run_dense_rows(di, p, Q, w, K, K_scale, T, N, H, d, q_pos0, 1, 0, (int64_t)T - 1, k, q_dtype, k_dtype,
                        idx, val, ws, nullptr, 0, st);
}

int dsa_debug_scores(const void* Q, const float* w, const void* K, const float* K_scale, int T, int N, int H, int d,
                     int64_t q_pos0, int q_dtype, int k_dtype, float* S, void* workspace, size_t workspace_bytes,
                     void* stream) {
  const int k = 1;
  int r = validate_dense(Q, w, K, K_scale, T, N, H, d, q_pos0, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (!S || !workspace) return DSA_ERR_INVALID_ARG;
  if ((int64_t)T * N > ((int64_t)1 << 26)) return DSA_ERR_UNSUPPORTED;
  DeviceInfo di;
  if ((r = device_info(di)) != DSA_OK) return r;
  Layout L;
  const size_t wo = take_widen(L, N, H, d, q_dtype, k_dtype);
  DensePlan p = plan_dense(di, T, N, H, d, q_dtype, k_dtype, L);
  // the top-1 outputs of this run go to scratch behind the plan
  const size_t oi = L.take((size_t)T * sizeof(int32_t));
  const size_t ov = L.take((size_t)T * sizeof(float));
  if (workspace_bytes < L.off) return DSA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((r = launch_fill_scores(S, (int64_t)T * N, st)) != DSA_OK) return r;
  const void* Kuse = K;
  int kd = k_dtype;
  if (needs_widen(H, d, q_dtype, k_dtype)) {
    if ((r = widen_keys(K, N, d, ws, wo, st)) != DSA_OK) return r;
    Kuse = ws + wo;
    kd = DSA_DTYPE_BF16;
  }
  return run_dense_rows(di, p, Q, w, Kuse, K_scale, T, N, H, d, q_pos0, 1, 0, (int64_t)T - 1, k, q_dtype, kd,
                        reinterpret_cast<int32_t*>(ws + oi), reinterpret_cast<float*>(ws + ov), ws, S, N, st);
}

}  // extern "C"

// --------------------------------------------------------------------------
// group and decode
// --------------------------------------------------------------------------
namespace {

struct GroupPlan {
  size_t widen_off;
  int ng;
  size_t qbar_off, wbar_off, bidx_off, bval_off, kg_off, map_off;
  int slots;            // refine key slots per group: bank + G (query-specific additions)
  DensePlan scan;       // proxy scan
  int64_t ref_cap;      // refine candidate capacity
  size_t ref_cand_off;
  int ref_grid;
  size_t total;
};

int plan_group(const DeviceInfo& di, int T, int N, int H, int d, int k, int G, int B, int q_dtype, int k_dtype,
               GroupPlan& gp) {
  Layout L;
  gp.widen_off = take_widen(L, N, H, d, q_dtype, k_dtype);
  gp.ng = (T + G - 1) / G;
  gp.qbar_off = L.take((size_t)gp.ng * H * d * elt_size(q_dtype));
  gp.wbar_off = L.take((size_t)gp.ng * H * sizeof(float));
  gp.bidx_off = L.take((size_t)gp.ng * B * sizeof(int32_t));
  gp.bval_off = L.take((size_t)gp.ng * B * sizeof(float));
  gp.scan = plan_dense(di, gp.ng, N, H, d, q_dtype, k_dtype, L);
  gp.kg_off = 0;
  gp.map_off = 0;
  gp.ref_cand_off = 0;
  gp.slots = B + G;
  gp.ref_cap = ((int64_t)gp.slots + 511) / 512 * 512;
  gp.ref_grid = 0;
  if (use_tc(H, d, q_dtype, k_dtype)) {
    gp.kg_off = L.take((size_t)gp.ng * gp.slots * d * 2);  // gathered bank keys, bf16
    gp.map_off = L.take((size_t)gp.ng * gp.slots * sizeof(int32_t));
    const int mblocks = (G + 3) / 4;
    const int64_t units = (int64_t)gp.ng * mblocks;
    gp.ref_grid = units < di.sms ? (int)units : di.sms;
    gp.ref_cand_off = L.take((size_t)gp.ref_grid * 4 * gp.ref_cap * sizeof(uint2));
  }
  gp.total = L.off;
  return DSA_OK;
}

}  // namespace

extern "C" {

int dsa_index_group_workspace_size(int T, int N, int H, int d, int k, int group, int bank, int q_dtype, int k_dtype,
                                   size_t* bytes) {
  if (!bytes) return DSA_ERR_INVALID_ARG;
  int r = check_common(H, d, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (T < 0 || N < 0 || group < 1 || bank < k || bank > kMaxBank) return DSA_ERR_INVALID_ARG;
  if (!use_tc(H, d, q_dtype, k_dtype)) return DSA_ERR_UNSUPPORTED;
  if (T == 0) return empty_workspace(bytes);
  if (N < 1) return DSA_ERR_INVALID_ARG;
  DeviceInfo di;
  if ((r = device_info(di)) != DSA_OK) return r;
  GroupPlan gp;
  plan_group(di, T, N, H, d, k, group, bank, q_dtype, k_dtype, gp);
  *bytes = gp.total;
  return DSA_OK;
}

int dsa_index_group(const void* Q, const float* w, const void* K, const float* K_scale, int T, int N, int H, int d,
                    int64_t q_pos0, int k, int group, int bank, int mode, int q_dtype, int k_dtype, int32_t* idx,
                    float* val, int32_t* bank_idx, float* bank_val, void* proxy_q, float* proxy_w, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (T == 0) {
    if (!group_args_ok(k, group, bank, mode)) return DSA_ERR_INVALID_ARG;
    return use_tc(H, d, q_dtype, k_dtype) ? empty_prefill(N, H, d, k, q_dtype, k_dtype, q_pos0) : DSA_ERR_UNSUPPORTED;
  }
  int r = validate_dense(Q, w, K, K_scale, T, N, H, d, q_pos0, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (!idx || !val || !workspace || group < 1 || bank < k || bank > kMaxBank) return DSA_ERR_INVALID_ARG;
  if (mode != DSA_GROUP_REFINE && mode != DSA_GROUP_REUSE && mode != DSA_GROUP_REFINE_LOCAL)
    return DSA_ERR_INVALID_ARG;
  if (!use_tc(H, d, q_dtype, k_dtype)) return DSA_ERR_UNSUPPORTED;
  if ((proxy_q && !aligned16(proxy_q)) || (proxy_w && !aligned16(proxy_w))) return DSA_ERR_INVALID_ARG;
  if (mode == DSA_GROUP_REFINE_LOCAL && group > 4096) return DSA_ERR_UNSUPPORTED;
  DeviceInfo di;
  if ((r = device_info(di)) != DSA_OK) return r;
  GroupPlan gp;
  plan_group(di, T, N, H, d, k, group, bank, q_dtype, k_dtype, gp);
  if (workspace_bytes < gp.total) return DSA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* qbar = proxy_q ? proxy_q : ws + gp.qbar_off;
  float* wbar = proxy_w ? proxy_w : reinterpret_cast<float*>(ws + gp.wbar_off);
  int32_t* bi = bank_idx ? bank_idx : reinterpret_cast<int32_t*>(ws + gp.bidx_off);
  float* bv = bank_val ? bank_val : reinterpret_cast<float*>(ws + gp.bval_off);
  // 0. fp8 keys: exact bf16 copy, the per-key scale goes to the epilogue
  if (needs_widen(H, d, q_dtype, k_dtype)) {
    if ((r = widen_keys(K, N, d, ws, gp.widen_off, st)) != DSA_OK) return r;
    K = ws + gp.widen_off;
    k_dtype = DSA_DTYPE_BF16;
  }
  // 1. proxies
  if ((r = launch_proxy_mean(Q, w, T, H, d, group, q_dtype, qbar, wbar, st)) != DSA_OK) return r;
  // 2. one full-prefix scan per proxy: bank = its top-`bank` keys
  if ((r = run_dense_rows(di, gp.scan, qbar, wbar, K, K_scale, gp.ng, N, H, d, q_pos0, group, group - 1,
                          (int64_t)T - 1, bank, q_dtype, k_dtype, bi, bv, ws, nullptr, 0, st)) != DSA_OK)
    return r;
  // 3. Reuse ranks the bank and finishes here.  Refine uses the bank as a
  // set; it is ranked only when the caller asked for it.
  const bool want_bank = bank_idx != nullptr || bank_val != nullptr;
  if (mode == DSA_GROUP_REUSE || want_bank) {
    if ((r = launch_bank_rank_reuse(bi, bv, gp.ng, bank, group, T, q_pos0, k, idx, val, mode == DSA_GROUP_REUSE,
                                    want_bank, st)) != DSA_OK)
      return r;
  }
  if (mode == DSA_GROUP_REUSE) return DSA_OK;
  // 4. Refine: members re-score their group's bank on tensor cores; with
  // query-specific additions each group's keys also follow its bank
  const bool local = mode == DSA_GROUP_REFINE_LOCAL;
  const int S = local ? bank + group : bank;
  const int32_t* kmap = bi;
  if (local) {
    int32_t* map = reinterpret_cast<int32_t*>(ws + gp.map_off);
    if ((r = launch_local_extend(bi, gp.ng, bank, group, T, q_pos0, nullptr, nullptr, S, map, st)) != DSA_OK)
      return r;
    kmap = map;
  }
  void* Kg = ws + gp.kg_off;
  if (!local && bank <= 8192) {
    // the bank in descending order of the proxy's score bin: members meet
    // their likely top keys first (the set, and so the results, unchanged)
    int32_t* map = reinterpret_cast<int32_t*>(ws + gp.map_off);
    if ((r = launch_bank_order_gather(K, bi, bv, gp.ng, bank, map, Kg, st)) != DSA_OK) return r;
    kmap = map;
  } else if ((r = launch_bank_gather(K, k_dtype, d, kmap, gp.ng, S, Kg, st)) != DSA_OK) {
    return r;
  }
  CUtensorMap tmQ, tmK;
  if ((r = make_map_bf16(&tmQ, Q, (uint64_t)T * H, (uint64_t)d, 64)) != DSA_OK) return r;
  if ((r = make_map_bf16(&tmK, Kg, (uint64_t)gp.ng * S, (uint64_t)d, 128)) != DSA_OK) return r;
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.kind = 2;
  a.k_scale = K_scale;
  a.n_rows = T;
  a.mblocks = (group + 3) / 4;
  a.n_units = gp.ng * a.mblocks;
  a.k = k;
  a.pos_base = q_pos0;
  a.w = w;
  a.out_idx = idx;
  a.out_val = val;
  a.out_ld = k;
  a.cand = reinterpret_cast<uint2*>(ws + gp.ref_cand_off);
  a.cand_cap = gp.ref_cap;
  a.status = reinterpret_cast<int*>(ws);
  a.key_map = kmap;
  a.bank = S;
  a.key_slots = local ? S : 0;
  a.group = group;
  a.T = T;
  return launch_tc_index(tmQ, tmK, a, gp.ref_grid, st);
}

}  // extern "C"

namespace {

struct DecodePlan {
  size_t widen_off;
  bool tc;
  int grid;
  int64_t cand_cap;
  int splits, tiles_per_split;
  size_t cand_off, ppair_off, pcnt_off, hdr_off, hist_off, total;
};

void plan_decode(const DeviceInfo& di, int B, int total_q, int64_t total_keys, int max_keys, int H, int d, int k,
                 int q_dtype, int k_dtype, DecodePlan& p) {
  memset(&p, 0, sizeof(p));
  p.tc = use_tc(H, d, q_dtype, k_dtype);
  Layout L;
  p.widen_off = take_widen(L, total_keys, H, d, q_dtype, k_dtype);
  const int tiles_max = (max_keys + 127) / 128;
  if (p.tc) {
    // split each cache into s pieces, s minimising (rounds of units over the
    // grid) x (tiles per unit + a per-unit cost of about 4 tiles)
    int best_s = 1;
    double best_cost = 1e300;
    for (int s = 1; s <= 256 && s <= tiles_max; ++s) {
      const int tps = (tiles_max + s - 1) / s;
      const int s_eff = (tiles_max + tps - 1) / tps;
      const int64_t units = (int64_t)B * s_eff;
      const int64_t rounds = (units + di.sms - 1) / di.sms;
      const double cost = (double)rounds * (tps + 4) + 0.01 * s_eff;
      if (cost < best_cost) {
        best_cost = cost;
        best_s = s_eff;
      }
    }
    p.splits = best_s;
    p.tiles_per_split = (tiles_max + best_s - 1) / best_s;
    p.cand_cap = (int64_t)((p.tiles_per_split + 3) / 4 * 4) * 128;
    const int64_t units = (int64_t)B * p.splits;
    p.grid = units < di.sms ? (int)units : di.sms;
    // every (row, slice) keeps its whole candidate list, segment header and
    // histogram for the merge
    const size_t lists = (size_t)total_q * p.splits;
    p.cand_off = L.take(lists * p.cand_cap * sizeof(uint2));
    p.hdr_off = L.take(lists * kSegHdr * sizeof(int));
    p.hist_off = L.take(lists * kBins * sizeof(uint32_t));
    p.total = L.off;
    return;
  } else {
    int s = (int)((2 * (int64_t)di.sms * 2 + total_q - 1) / total_q);
    if (s < 1) s = 1;
    if (s > 256) s = 256;
    if (s > tiles_max) s = tiles_max;
    const int kps = (int)((((int64_t)max_keys + s - 1) / s + 127) / 128 * 128);
    p.tiles_per_split = kps / 128;
    p.splits = (int)(((int64_t)max_keys + kps - 1) / kps);
    p.cand_cap = kps;
    p.grid = simt_grid(di, (int64_t)total_q * p.splits);
    p.cand_off = L.take((size_t)p.grid * 2 * p.cand_cap * sizeof(uint2));
  }
  const size_t parts = (size_t)total_q * p.splits;
  p.ppair_off = L.take(parts * k * sizeof(uint2));
  p.pcnt_off = L.take(parts * sizeof(int));
  p.total = L.off;
}

// Tensor-core decode scan of `rows` query rows (q_offsets == nullptr: one row
// per sequence), whose slices leave their whole candidate lists, followed by
// the merge that selects each row's top k from them into idx / val [rows, k].
// K is bf16 (fp8 keys already widened).
int run_decode_tc(const DecodePlan& p, const void* Q, const float* w, const void* K, const float* K_scale,
                  const int64_t* k_offsets, const int32_t* q_offsets, int B, int rows, int64_t total_keys, int H,
                  int d, int k, int32_t* idx, float* val, uint8_t* ws, cudaStream_t st, const int* ok = nullptr) {
  int r;
  uint2* cand = reinterpret_cast<uint2*>(ws + p.cand_off);
  int* hdr = reinterpret_cast<int*>(ws + p.hdr_off);
  uint32_t* hist = reinterpret_cast<uint32_t*>(ws + p.hist_off);
  int* status = reinterpret_cast<int*>(ws);
  CUtensorMap tmQ, tmK;
  if ((r = make_map_bf16(&tmQ, Q, (uint64_t)rows * H, (uint64_t)d, 64)) != DSA_OK) return r;
  // rows: the whole key array; a tile running past its sequence's end is
  // masked per key, and rows past the array's end read as zeros
  if ((r = make_map_bf16(&tmK, K, (uint64_t)total_keys, (uint64_t)d, 128)) != DSA_OK) return r;
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.kind = 1;
  a.k_scale = K_scale;
  a.n_rows = rows;
  a.n_units = B * p.splits;
  a.k = k;
  a.w = w;
  a.out_ld = k;
  a.out_cnt = hdr;
  a.out_hist = hist;
  a.cand = cand;
  a.cand_cap = p.cand_cap;
  a.status = status;
  a.k_off = k_offsets;
  a.q_off = q_offsets;
  a.splits = p.splits;
  a.tiles_per_split = p.tiles_per_split;
  a.total_keys = total_keys;
  a.offsets_ok = ok;
  if ((r = launch_tc_index(tmQ, tmK, a, p.grid, st)) != DSA_OK) return r;
  return launch_decode_merge_lists(cand, p.cand_cap, hdr, hist, rows, p.splits, k, idx, val, status, st, ok);
}

}  // namespace

extern "C" {

int dsa_index_decode_workspace_size(int B, int total_q, int max_keys, int H, int d, int k, int q_dtype, int k_dtype,
                                    size_t* bytes) {
  if (!bytes) return DSA_ERR_INVALID_ARG;
  int r = check_common(H, d, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (B < 0 || total_q < 0 || max_keys < 0) return DSA_ERR_INVALID_ARG;
  if (B == 0) return total_q == 0 ? empty_workspace(bytes) : DSA_ERR_INVALID_ARG;
  if (total_q < 1 || max_keys < 1) return DSA_ERR_INVALID_ARG;
  DeviceInfo di;
  if ((r = device_info(di)) != DSA_OK) return r;
  DecodePlan p;
  plan_decode(di, B, total_q, (int64_t)B * max_keys, max_keys, H, d, k, q_dtype, k_dtype, p);
  *bytes = p.total;
  return DSA_OK;
}

int dsa_index_decode(const void* Q, const float* w, const void* K, const float* K_scale, const int64_t* k_offsets,
                     const int32_t* q_offsets, int B, int total_q, int64_t total_keys, int max_keys, int H, int d,
                     int k, int q_dtype, int k_dtype, int32_t* idx, float* val, void* workspace,
                     size_t workspace_bytes, void* stream) {
  if (B == 0) return empty_decode(total_q, total_keys, H, d, k, q_dtype, k_dtype);
  int r = check_common(H, d, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (!Q || !w || !K || !k_offsets || !q_offsets || !idx || !val || !workspace) return DSA_ERR_INVALID_ARG;
  if (B < 1 || total_q < 1 || max_keys < 1 || total_keys < 1 || max_keys > total_keys) return DSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(w)) return DSA_ERR_INVALID_ARG;
  if ((k_dtype == DSA_DTYPE_FP8_E4M3) != (K_scale != nullptr)) return DSA_ERR_INVALID_ARG;
  // the tensor-core kernel addresses key rows with 32-bit TMA coordinates
  if (use_tc(H, d, q_dtype, k_dtype) && total_keys > ((int64_t)1 << 31) - 256) return DSA_ERR_UNSUPPORTED;
  DeviceInfo di;
  if ((r = device_info(di)) != DSA_OK) return r;
  DecodePlan p;
  plan_decode(di, B, total_q, total_keys, max_keys, H, d, k, q_dtype, k_dtype, p);
  if (workspace_bytes < p.total) return DSA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (needs_widen(H, d, q_dtype, k_dtype)) {
    if ((r = widen_keys(K, total_keys, d, ws, p.widen_off, st)) != DSA_OK) return r;
    K = ws + p.widen_off;
  }
  if (p.tc)
    return run_decode_tc(p, Q, w, K, K_scale, k_offsets, q_offsets, B, total_q, total_keys, H, d, k, idx, val, ws, st);
  int* status = reinterpret_cast<int*>(ws);
  uint2* ppair = reinterpret_cast<uint2*>(ws + p.ppair_off);
  int* pcnt = reinterpret_cast<int*>(ws + p.pcnt_off);
  {
    SimtArgs a;
    memset(&a, 0, sizeof(a));
    a.kind = 1;
    a.n_tasks = total_q * p.splits;
    a.H = H;
    a.d = d;
    a.k = k;
    a.q_dtype = q_dtype;
    a.k_dtype = k_dtype;
    a.Q = Q;
    a.w = w;
    a.K = K;
    a.K_scale = K_scale;
    a.out_pair = ppair;
    a.out_ld = k;
    a.out_cnt = pcnt;
    a.cand = reinterpret_cast<uint2*>(ws + p.cand_off);
    a.cand_cap = p.cand_cap;
    a.status = status;
    a.k_off = k_offsets;
    a.q_off = q_offsets;
    a.B = B;
    a.splits = p.splits;
    a.keys_per_split = p.tiles_per_split * 128;
    a.total_keys = total_keys;
    if ((r = launch_simt_index(a, p.grid, st)) != DSA_OK) return r;
  }
  return launch_decode_merge(ppair, pcnt, total_q, p.splits, k, idx, val, status, st);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// PIVOT in decode: each sequence's new queries are one group.
// ---------------------------------------------------------------------------
namespace {

struct DecodeGroupPlan {
  DecodePlan scan;  // the proxies' cache scan: one row per sequence, k = bank
  size_t qbar_off, wbar_off, bidx_off, bval_off, kg_off, map_off, ref_cand_off, total;
  int slots;  // refine key slots per sequence: bank + 4 (query-specific additions)
  int ref_grid;
  int64_t ref_cap;
};

void plan_decode_group(const DeviceInfo& di, int B, int64_t total_keys, int max_keys, int H, int d, int bank,
                       int q_dtype, int k_dtype, DecodeGroupPlan& gp) {
  plan_decode(di, B, B, total_keys, max_keys, H, d, bank, q_dtype, k_dtype, gp.scan);
  Layout L;
  L.off = gp.scan.total;
  gp.qbar_off = L.take((size_t)B * H * d * 2);
  gp.wbar_off = L.take((size_t)B * H * sizeof(float));
  gp.bidx_off = L.take((size_t)B * bank * sizeof(int32_t));
  gp.bval_off = L.take((size_t)B * bank * sizeof(float));
  gp.slots = bank + 4;
  gp.kg_off = L.take((size_t)B * gp.slots * d * 2);
  gp.map_off = L.take((size_t)B * gp.slots * sizeof(int32_t));
  // refine: one unit per sequence (m_b <= 4 queries), candidate lists as for
  // the prefill refine (whole groups of 4 key tiles)
  gp.ref_cap = ((int64_t)gp.slots + 511) / 512 * 512;
  gp.ref_grid = B < di.sms ? B : di.sms;
  gp.ref_cand_off = L.take((size_t)gp.ref_grid * 4 * gp.ref_cap * sizeof(uint2));
  gp.total = L.off;
}

}  // namespace

extern "C" {

int dsa_index_decode_group_workspace_size(int B, int total_q, int max_keys, int H, int d, int k, int bank,
                                          int q_dtype, int k_dtype, size_t* bytes) {
  if (!bytes) return DSA_ERR_INVALID_ARG;
  int r = check_common(H, d, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (B < 0 || total_q < 0 || max_keys < 0 || bank < k || bank > kMaxBank) return DSA_ERR_INVALID_ARG;
  if (!use_tc(H, d, q_dtype, k_dtype)) return DSA_ERR_UNSUPPORTED;
  if (B == 0) return total_q == 0 ? empty_workspace(bytes) : DSA_ERR_INVALID_ARG;
  if (total_q < 1 || max_keys < 1) return DSA_ERR_INVALID_ARG;
  DeviceInfo di;
  if ((r = device_info(di)) != DSA_OK) return r;
  DecodeGroupPlan gp;
  plan_decode_group(di, B, (int64_t)B * max_keys, max_keys, H, d, bank, q_dtype, k_dtype, gp);
  *bytes = gp.total;
  return DSA_OK;
}

int dsa_index_decode_group(const void* Q, const float* w, const void* K, const float* K_scale,
                           const int64_t* k_offsets, const int32_t* q_offsets, int B, int total_q, int64_t total_keys,
                           int max_keys, int H, int d, int k, int bank, int mode, int q_dtype, int k_dtype,
                           int32_t* idx, float* val, int32_t* bank_idx, float* bank_val, void* proxy_q,
                           float* proxy_w, void* workspace, size_t workspace_bytes, void* stream) {
  if (B == 0) {
    if (!group_args_ok(k, 1, bank, mode)) return DSA_ERR_INVALID_ARG;
    if (!use_tc(H, d, q_dtype, k_dtype)) return DSA_ERR_UNSUPPORTED;
    return empty_decode(total_q, total_keys, H, d, k, q_dtype, k_dtype);
  }
  int r = check_common(H, d, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (!Q || !w || !K || !k_offsets || !q_offsets || !idx || !val || !workspace) return DSA_ERR_INVALID_ARG;
  if (B < 1 || total_q < 1 || max_keys < 1 || total_keys < 1 || max_keys > total_keys) return DSA_ERR_INVALID_ARG;
  if (bank < k || bank > kMaxBank) return DSA_ERR_INVALID_ARG;
  if (mode != DSA_GROUP_REFINE && mode != DSA_GROUP_REUSE && mode != DSA_GROUP_REFINE_LOCAL)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(w)) return DSA_ERR_INVALID_ARG;
  if ((proxy_q && !aligned16(proxy_q)) || (proxy_w && !aligned16(proxy_w))) return DSA_ERR_INVALID_ARG;
  if ((k_dtype == DSA_DTYPE_FP8_E4M3) != (K_scale != nullptr)) return DSA_ERR_INVALID_ARG;
  if (!use_tc(H, d, q_dtype, k_dtype)) return DSA_ERR_UNSUPPORTED;
  if (total_keys > ((int64_t)1 << 31) - 256) return DSA_ERR_UNSUPPORTED;
  DeviceInfo di;
  if ((r = device_info(di)) != DSA_OK) return r;
  DecodeGroupPlan gp;
  plan_decode_group(di, B, total_keys, max_keys, H, d, bank, q_dtype, k_dtype, gp);
  if (workspace_bytes < gp.total) return DSA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* qbar = proxy_q ? proxy_q : ws + gp.qbar_off;
  float* wbar = proxy_w ? proxy_w : reinterpret_cast<float*>(ws + gp.wbar_off);
  int32_t* bi = bank_idx ? bank_idx : reinterpret_cast<int32_t*>(ws + gp.bidx_off);
  float* bv = bank_val ? bank_val : reinterpret_cast<float*>(ws + gp.bval_off);
  // 0. the offsets, checked once on the device: every later kernel that
  // reads them does nothing if they failed (invalid argument in the status)
  if ((r = launch_decode_offsets_check(k_offsets, q_offsets, B, total_keys, total_q, max_keys, ws, st)) != DSA_OK)
    return r;
  const int* ok = &reinterpret_cast<const WsHeader*>(ws)->offsets_ok;
  // fp8 keys: exact bf16 copy, the per-key scale goes to the epilogue
  if (needs_widen(H, d, q_dtype, k_dtype)) {
    if ((r = widen_keys(K, total_keys, d, ws, gp.scan.widen_off, st)) != DSA_OK) return r;
    K = ws + gp.scan.widen_off;
  }
  // 1. proxies: the mean of each sequence's new queries
  if ((r = launch_proxy_mean(Q, w, total_q, H, d, 1, q_dtype, qbar, wbar, st, q_offsets, B, ok)) != DSA_OK) return r;
  // 2. one scan of each cache by its proxy, which sits at the last query's
  // position N_b - 1: bank = its top-`bank` keys (local indices)
  if ((r = run_decode_tc(gp.scan, qbar, wbar, K, K_scale, k_offsets, nullptr, B, B, total_keys, H, d, bank, bi, bv,
                         ws, st, ok)) != DSA_OK)
    return r;
  // 3. Reuse ranks the bank and finishes here; Refine ranks it only for the
  // caller's bank output.  A sequence's queries drop at most 3 bank keys
  // (m_b <= 4), so Reuse needs the top k + 3.
  const bool want_bank = bank_idx != nullptr || bank_val != nullptr;
  if (mode == DSA_GROUP_REUSE || want_bank) {
    if ((r = launch_bank_rank_reuse(bi, bv, B, bank, 4, total_q, 0, k, idx, val, mode == DSA_GROUP_REUSE, want_bank,
                                    st, q_offsets, k_offsets, ok)) != DSA_OK)
      return r;
  }
  if (mode == DSA_GROUP_REUSE) return DSA_OK;
  // 4. Refine: each sequence's queries re-score its bank on tensor cores;
  // with query-specific additions the sequence's new keys follow its bank
  const bool local = mode == DSA_GROUP_REFINE_LOCAL;
  const int S = local ? gp.slots : bank;
  const int32_t* kmap = bi;
  if (local) {
    int32_t* map = reinterpret_cast<int32_t*>(ws + gp.map_off);
    if ((r = launch_local_extend(bi, B, bank, 4, total_q, 0, q_offsets, k_offsets, S, map, st, ok)) != DSA_OK)
      return r;
    kmap = map;
  }
  void* Kg = ws + gp.kg_off;
  if ((r = launch_bank_gather(K, DSA_DTYPE_BF16, d, kmap, B, S, Kg, st, k_offsets, ok)) != DSA_OK) return r;
  CUtensorMap tmQ, tmK;
  if ((r = make_map_bf16(&tmQ, Q, (uint64_t)total_q * H, (uint64_t)d, 64)) != DSA_OK) return r;
  if ((r = make_map_bf16(&tmK, Kg, (uint64_t)B * S, (uint64_t)d, 128)) != DSA_OK) return r;
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.kind = 2;
  a.k_scale = K_scale;
  a.n_rows = total_q;
  a.mblocks = 1;
  a.n_units = B;
  a.k = k;
  a.w = w;
  a.out_idx = idx;
  a.out_val = val;
  a.out_ld = k;
  a.cand = reinterpret_cast<uint2*>(ws + gp.ref_cand_off);
  a.cand_cap = gp.ref_cap;
  a.status = reinterpret_cast<int*>(ws);
  a.key_map = kmap;
  a.bank = S;
  a.key_slots = local ? S : 0;
  a.T = total_q;
  a.k_off = k_offsets;
  a.q_off = q_offsets;
  a.total_keys = total_keys;
  a.offsets_ok = ok;
  return launch_tc_index(tmQ, tmK, a, gp.ref_grid, st);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Two-stage selection over contiguous blocks (block routing) with the native
// score on the routed keys.
// ---------------------------------------------------------------------------
namespace {

struct RoutedPlan {
  size_t widen_off, reps_off, bidx_off, bval_off, ref_cand_off, total;
  int64_t nblocks;
  DensePlan route;  // the queries against the block representatives
  int ref_grid;
  int64_t ref_cap;
};

void plan_routed(const DeviceInfo& di, int T, int N, int H, int d, int n_blocks, int q_dtype, int k_dtype,
                 RoutedPlan& p) {
  Layout L;
  p.widen_off = take_widen(L, N, H, d, q_dtype, k_dtype);
  p.nblocks = ((int64_t)N + 127) / 128;
  p.reps_off = L.take((size_t)p.nblocks * d * 2);
  p.bidx_off = L.take((size_t)T * n_blocks * sizeof(int32_t));
  p.bval_off = L.take((size_t)T * n_blocks * sizeof(float));
  p.route = plan_dense(di, T, (int)p.nblocks, H, d, q_dtype, DSA_DTYPE_BF16, L);
  // refine: one query per unit over at most n_blocks + 1 tiles (whole groups of 4)
  p.ref_cap = ((int64_t)n_blocks + 1 + 3) / 4 * 4 * 128;
  p.ref_grid = T < di.sms ? T : di.sms;
  p.ref_cand_off = L.take((size_t)p.ref_grid * 4 * p.ref_cap * sizeof(uint2));
  p.total = L.off;
}

}  // namespace

extern "C" {

int dsa_index_block_routed_workspace_size(int T, int N, int H, int d, int k, int n_blocks, int q_dtype,
                                          int k_dtype, size_t* bytes) {
  if (!bytes) return DSA_ERR_INVALID_ARG;
  int r = check_common(H, d, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (T < 0 || N < 0 || n_blocks < 1 || n_blocks > 65536) return DSA_ERR_INVALID_ARG;
  if (!use_tc(H, d, q_dtype, k_dtype)) return DSA_ERR_UNSUPPORTED;
  if (T == 0) return empty_workspace(bytes);
  if (N < 1) return DSA_ERR_INVALID_ARG;
  DeviceInfo di;
  if ((r = device_info(di)) != DSA_OK) return r;
  RoutedPlan p;
  plan_routed(di, T, N, H, d, n_blocks, q_dtype, k_dtype, p);
  *bytes = p.total;
  return DSA_OK;
}

int dsa_index_block_routed(const void* Q, const float* w, const void* K, const float* K_scale, int T, int N, int H,
                           int d, int64_t q_pos0, int k, int n_blocks, int q_dtype, int k_dtype, int32_t* idx,
                           float* val, int32_t* block_idx, void* reps, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (T == 0) {
    if (n_blocks < 1 || n_blocks > 65536) return DSA_ERR_INVALID_ARG;
    return use_tc(H, d, q_dtype, k_dtype) ? empty_prefill(N, H, d, k, q_dtype, k_dtype, q_pos0) : DSA_ERR_UNSUPPORTED;
  }
  int r = validate_dense(Q, w, K, K_scale, T, N, H, d, q_pos0, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (!idx || !val || !workspace || n_blocks < 1 || n_blocks > 65536) return DSA_ERR_INVALID_ARG;
  if (!use_tc(H, d, q_dtype, k_dtype)) return DSA_ERR_UNSUPPORTED;
  if (reps && !aligned16(reps)) return DSA_ERR_INVALID_ARG;
  DeviceInfo di;
  if ((r = device_info(di)) != DSA_OK) return r;
  RoutedPlan p;
  plan_routed(di, T, N, H, d, n_blocks, q_dtype, k_dtype, p);
  if (workspace_bytes < p.total) return DSA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (needs_widen(H, d, q_dtype, k_dtype)) {
    if ((r = widen_keys(K, N, d, ws, p.widen_off, st)) != DSA_OK) return r;
    K = ws + p.widen_off;
  }
  // 1. block representatives (fp8 keys: the mean of the scaled keys)
  void* R = reps ? reps : ws + p.reps_off;
  if ((r = launch_block_mean(K, K_scale, N, d, R, st)) != DSA_OK) return r;
  // 2. routing: each query's best n_blocks complete blocks before it
  int32_t* bi = block_idx ? block_idx : reinterpret_cast<int32_t*>(ws + p.bidx_off);
  float* bv = reinterpret_cast<float*>(ws + p.bval_off);
  if ((r = run_dense_rows(di, p.route, Q, w, R, nullptr, T, (int)p.nblocks, H, d, q_pos0, 1, 0, (int64_t)T, n_blocks,
                          q_dtype, DSA_DTYPE_BF16, bi, bv, ws, nullptr, 0, st, 7)) != DSA_OK)  // 128-key blocks
    return r;
  // 3. refine: the native score over the routed blocks and the own partial block
  CUtensorMap tmQ, tmK;
  if ((r = make_map_bf16(&tmQ, Q, (uint64_t)T * H, (uint64_t)d, 64)) != DSA_OK) return r;
  if ((r = make_map_bf16(&tmK, K, (uint64_t)N, (uint64_t)d, 128)) != DSA_OK) return r;
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.kind = 3;
  a.k_scale = K_scale;
  a.n_rows = T;
  a.n_units = T;
  a.k = k;
  a.pos_base = q_pos0;
  a.w = w;
  a.out_idx = idx;
  a.out_val = val;
  a.out_ld = k;
  a.cand = reinterpret_cast<uint2*>(ws + p.ref_cand_off);
  a.cand_cap = p.ref_cap;
  a.status = reinterpret_cast<int*>(ws);
  a.route_blocks = bi;
  a.route_n = n_blocks;
  return launch_tc_index(tmQ, tmK, a, p.ref_grid, st);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Inverted-file routing: plain k-means index, then the native score on the
// probed clusters' keys.
// ---------------------------------------------------------------------------
namespace {

struct IvfPlan {
  size_t widen_off, scratch_off, cidx_off, cval_off, tiles_off, ref_cand_off, total;
  DensePlan route;  // the queries against the centroids
  int ref_grid;
  int64_t ref_cap;
};

// Build workspace: the widened keys (fp8) and the k-means sums.
size_t ivf_build_workspace(int64_t N, int H, int d, int C, int q_dtype, int k_dtype) {
  Layout L;
  take_widen(L, N, H, d, q_dtype, k_dtype);
  L.take(ivf_build_scratch_bytes(d, C));
  return L.off;
}

void plan_ivf(const DeviceInfo& di, int T, int N, int H, int d, int C, int n_probe, int64_t max_tiles, int q_dtype,
              IvfPlan& p) {
  Layout L;
  p.widen_off = 0;
  p.scratch_off = 0;
  p.cidx_off = L.take((size_t)T * n_probe * sizeof(int32_t));
  p.cval_off = L.take((size_t)T * n_probe * sizeof(float));
  p.tiles_off = L.take((size_t)T * sizeof(int32_t));
  p.route = plan_dense(di, T, C, H, d, q_dtype, DSA_DTYPE_BF16, L);
  // refine: one query per unit over at most max_tiles tiles (whole groups of 4)
  p.ref_cap = (max_tiles + 3) / 4 * 4 * 128;
  p.ref_grid = T < di.sms ? T : di.sms;
  p.ref_cand_off = L.take((size_t)p.ref_grid * 4 * p.ref_cap * sizeof(uint2));
  p.total = L.off;
}

}  // namespace

extern "C" {

int dsa_ivf_index_size(int N, int d, int C, size_t* bytes) {
  if (!bytes || N < 1 || d < 32 || d > 256 || d % 32 || C < 1 || C > N || C > 65536) return DSA_ERR_INVALID_ARG;
  *bytes = ivf_index_view(nullptr, N, d, C).bytes;
  return DSA_OK;
}

int dsa_ivf_build_workspace_size(int N, int H, int d, int C, int q_dtype, int k_dtype, size_t* bytes) {
  if (!bytes || N < 1 || C < 1 || C > N || C > 65536) return DSA_ERR_INVALID_ARG;
  int r = check_common(H, d, 1, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (!use_tc(H, d, q_dtype, k_dtype)) return DSA_ERR_UNSUPPORTED;
  *bytes = ivf_build_workspace(N, H, d, C, q_dtype, k_dtype);
  return DSA_OK;
}

int dsa_ivf_build(const void* K, const float* K_scale, int N, int H, int d, int C, int iters, int q_dtype,
                  int k_dtype, void* index, size_t index_bytes, void* workspace, size_t workspace_bytes,
                  void* stream) {
  int r = check_common(H, d, 1, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (!K || !index || !workspace || N < 1 || C < 1 || C > N || C > 65536 || iters < 1 || iters > 1000)
    return DSA_ERR_INVALID_ARG;
  if ((k_dtype == DSA_DTYPE_FP8_E4M3) != (K_scale != nullptr)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(index)) return DSA_ERR_INVALID_ARG;
  if (!use_tc(H, d, q_dtype, k_dtype)) return DSA_ERR_UNSUPPORTED;
  DeviceInfo di;
  if ((r = device_info(di)) != DSA_OK) return r;
  const IvfIndex x = ivf_index_view(index, N, d, C);
  if (index_bytes < x.bytes) return DSA_ERR_WORKSPACE;
  if (workspace_bytes < ivf_build_workspace(N, H, d, C, q_dtype, k_dtype)) return DSA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Layout L;
  const size_t widen_off = take_widen(L, N, H, d, q_dtype, k_dtype);
  const size_t scratch_off = L.take(ivf_build_scratch_bytes(d, C));
  if (needs_widen(H, d, q_dtype, k_dtype)) {
    if ((r = widen_keys(K, N, d, ws, widen_off, st)) != DSA_OK) return r;
    K = ws + widen_off;
  }
  return ivf_build(K, K_scale, N, d, C, iters, x, ws + scratch_off, st);
}

int dsa_index_ivf_routed_workspace_size(int T, int N, int H, int d, int k, int C, int n_probe, int max_tiles,
                                        int q_dtype, int k_dtype, size_t* bytes) {
  if (!bytes) return DSA_ERR_INVALID_ARG;
  int r = check_common(H, d, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (T < 0 || N < 1 || C < 1 || n_probe < 1 || n_probe > C || max_tiles < 1) return DSA_ERR_INVALID_ARG;
  if (!use_tc(H, d, q_dtype, k_dtype)) return DSA_ERR_UNSUPPORTED;
  if (T == 0) return empty_workspace(bytes);
  DeviceInfo di;
  if ((r = device_info(di)) != DSA_OK) return r;
  IvfPlan p;
  plan_ivf(di, T, N, H, d, C, n_probe, max_tiles, q_dtype, p);
  *bytes = p.total;
  return DSA_OK;
}

int dsa_index_ivf_routed(const void* Q, const float* w, const void* index, const float* K_scale, int T, int N,
                         int H, int d, int64_t q_pos0, int k, int C, int n_probe, int max_tiles, int q_dtype,
                         int k_dtype, int32_t* idx, float* val, int32_t* cluster_idx, void* workspace,
                         size_t workspace_bytes, void* stream) {
  if (T == 0) {
    if (N < 1 || C < 1 || C > N || n_probe < 1 || n_probe > C || max_tiles < 1) return DSA_ERR_INVALID_ARG;
    return use_tc(H, d, q_dtype, k_dtype) ? empty_prefill(N, H, d, k, q_dtype, k_dtype, q_pos0) : DSA_ERR_UNSUPPORTED;
  }
  int r = check_common(H, d, k, q_dtype, k_dtype);
  if (r != DSA_OK) return r;
  if (!Q || !w || !index || !idx || !val || !workspace) return DSA_ERR_INVALID_ARG;
  if (T < 1 || N < 1 || q_pos0 < 0 || q_pos0 + (int64_t)T > (int64_t)N) return DSA_ERR_INVALID_ARG;
  if (C < 1 || C > N || n_probe < 1 || n_probe > C || max_tiles < 1) return DSA_ERR_INVALID_ARG;
  if ((k_dtype == DSA_DTYPE_FP8_E4M3) != (K_scale != nullptr)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(w) || !aligned16(index)) return DSA_ERR_INVALID_ARG;
  if (!use_tc(H, d, q_dtype, k_dtype)) return DSA_ERR_UNSUPPORTED;
  DeviceInfo di;
  if ((r = device_info(di)) != DSA_OK) return r;
  IvfPlan p;
  plan_ivf(di, T, N, H, d, C, n_probe, max_tiles, q_dtype, p);
  if (workspace_bytes < p.total) return DSA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const IvfIndex x = ivf_index_view(const_cast<void*>(index), N, d, C);
  // 1. routing: every centroid is visible to every query (pos = C - 1)
  int32_t* ci = cluster_idx ? cluster_idx : reinterpret_cast<int32_t*>(ws + p.cidx_off);
  float* cv = reinterpret_cast<float*>(ws + p.cval_off);
  if ((r = run_dense_rows(di, p.route, Q, w, x.cen_bf16, nullptr, T, C, H, d, C - 1, 0, 0, 0, n_probe, q_dtype,
                          DSA_DTYPE_BF16, ci, cv, ws, nullptr, 0, st)) != DSA_OK)
    return r;
  // 2. the tiles each query streams, then the refine over its clusters' keys
  int32_t* tiles = reinterpret_cast<int32_t*>(ws + p.tiles_off);
  if ((r = launch_ivf_tiles(ci, n_probe, T, x.off, tiles, st)) != DSA_OK) return r;
  CUtensorMap tmQ, tmK;
  if ((r = make_map_bf16(&tmQ, Q, (uint64_t)T * H, (uint64_t)d, 64)) != DSA_OK) return r;
  if ((r = make_map_bf16(&tmK, x.keys, (uint64_t)N, (uint64_t)d, 128)) != DSA_OK) return r;
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.kind = 4;
  a.k_scale = K_scale;
  a.n_rows = T;
  a.n_units = T;
  a.k = k;
  a.pos_base = q_pos0;
  a.w = w;
  a.out_idx = idx;
  a.out_val = val;
  a.out_ld = k;
  a.cand = reinterpret_cast<uint2*>(ws + p.ref_cand_off);
  a.cand_cap = p.ref_cap;
  a.status = reinterpret_cast<int*>(ws);
  a.key_map = x.perm;
  a.route_blocks = ci;
  a.route_n = n_probe;
  a.ivf_off = x.off;
  a.ivf_tiles = tiles;
  a.ivf_max_tiles = max_tiles;
  return launch_tc_index(tmQ, tmK, a, p.ref_grid, st);
}

}  // extern "C"
