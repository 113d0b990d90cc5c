// dsa_static.cu — dense indexer entry point that allocates nothing.
//
// Some callers cannot hand this library a workspace: code that runs inside a
// host application which reserved all device memory for itself up front (a
// serving engine that sizes its KV cache to the whole GPU, for instance), or
// a real-time loop where a late cudaMalloc may fail under memory pressure or
// stall the device.  For them, dsa_index_dense_static runs the same
// tensor-core kernel as dsa_index_dense with its scratch (status word and
// per-CTA candidate lists) in a fixed array in device memory that this
// library reserves when it is loaded.  The caller still provides Q, w, K and
// the outputs.
#include <cstring>
#include <mutex>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace {

// Fixed scratch: 32 MiB on every GPU that loads the library, held until the
// process exits.  Layout: a 256-byte status header, then the candidate lists.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
// Device address of g_static_scratch per device, with the context it was
// resolved in: a device reset makes a new context (and loads the module
// again), so the address is resolved once per device and context.
void* g_scratch_ptr[kMaxDevices];
CUcontext g_scratch_ctx[kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// With the device current: the device address of the array (its host-side
// name is only a stand-in, not a device address).
int scratch_address(int dev, void** out) {
  static CtxGetCurrentFn ctx_fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] { ctx_fn = reinterpret_cast<CtxGetCurrentFn>(dsa::driver_entry("cuCtxGetCurrent")); });
  CUcontext ctx = nullptr;
  if (!ctx_fn || ctx_fn(&ctx) != CUDA_SUCCESS || ctx == nullptr) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return DSA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return DSA_OK;
}

}  // namespace

extern "C" int dsa_index_dense_static(const void* Q, const float* w, const void* K, int T, int N, int H, int d,
                                      int64_t q_pos0, int k, int32_t* idx, float* val, void* stream) {
  if (T == 0) {  // no query rows: nothing to compute, nothing launched
    if (N < 0 || q_pos0 < 0 || q_pos0 > (int64_t)N || k < 1 || k > 65536) return DSA_ERR_INVALID_ARG;
    return (H != 64 || d != 128) ? DSA_ERR_UNSUPPORTED : DSA_OK;
  }
  if (!Q || !w || !K || !idx || !val) return DSA_ERR_INVALID_ARG;
  if (T < 1 || N < 1 || q_pos0 < 0 || q_pos0 + (int64_t)T > (int64_t)N || k < 1 || k > 65536)
    return DSA_ERR_INVALID_ARG;
  if (((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(w)) & 15u) != 0)
    return DSA_ERR_INVALID_ARG;
  if (H != 64 || d != 128) return DSA_ERR_UNSUPPORTED;  // bf16 tensor-core shape only
  int dev = 0, sms = 0;
  int r = dsa::current_device(&dev, &sms);  // compute capability 10.0, as every entry
  if (r != DSA_OK) return r;
  if (dev >= kMaxDevices) return DSA_ERR_DEVICE;

  // Each CTA of the kernel keeps 4 candidate lists of round_up(N, 512)
  // entries (whole groups of 4 key tiles); the grid shrinks to what the
  // fixed scratch holds.
  const int64_t cap = ((int64_t)N + 511) / 512 * 512;
  const size_t per_cta = (size_t)4 * cap * sizeof(uint2);
  const int units = (T + 3) / 4;
  const int64_t fit = (int64_t)((kStaticScratchBytes - 256) / per_cta);
  if (fit < 1) return DSA_ERR_WORKSPACE;  // N too large for the fixed scratch
  int grid = units < sms ? units : sms;
  if (grid > fit) grid = (int)fit;

  void* base = nullptr;
  if ((r = scratch_address(dev, &base)) != DSA_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the status word must start at zero; candidate lists need no clearing
  if (cudaMemsetAsync(base, 0, 256, st) != cudaSuccess) return DSA_ERR_CUDA;

  CUtensorMap tmQ, tmK;
  if ((r = dsa::make_map_bf16(&tmQ, Q, (uint64_t)T * H, (uint64_t)d, 64)) != DSA_OK) return r;
  if ((r = dsa::make_map_bf16(&tmK, K, (uint64_t)N, (uint64_t)d, 128)) != DSA_OK) return r;
  dsa::TcArgs a;
  memset(&a, 0, sizeof(a));
  a.kind = 0;
  a.n_rows = T;
  a.n_units = units;
  a.k = k;
  a.pos_base = q_pos0;
  a.pos_mul = 1;
  a.pos_add = 0;
  a.pos_clamp = (int64_t)T - 1;
  a.w = w;
  a.out_idx = idx;
  a.out_val = val;
  a.out_ld = k;
  a.cand = reinterpret_cast<uint2*>(static_cast<unsigned char*>(base) + 256);
  a.cand_cap = cap;
  a.status = static_cast<int*>(base);
  if ((r = dsa::launch_tc_index(tmQ, tmK, a, grid, st)) != DSA_OK) return r;
  // wait for this call and report a device-side failure it recorded
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  int status = 0;
  if (cudaMemcpy(&status, base, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return DSA_ERR_CUDA;
  return status;
}
