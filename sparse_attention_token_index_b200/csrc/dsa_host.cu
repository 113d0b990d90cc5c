// Host-buffer entry points: the dense, group and decode indexers called with
// inputs and outputs in host memory.  The inputs are staged into a device
// buffer the caller owns; dense and group calls run in row chunks so that the
// host-to-device copy of chunk c+1, the indexer on chunk c and the
// device-to-host copy of chunk c-1 overlap (copies on two library streams,
// the indexer on the caller's stream, ordered by per-chunk events).
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "dsa_index.h"

namespace {

constexpr int kMaxChunks = 64;

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t elem_size(int dtype) {
  switch (dtype) {
    case DSA_DTYPE_BF16: return 2;
    case DSA_DTYPE_FP32: return 4;
    case DSA_DTYPE_FP8_E4M3: return 1;
    default: return 0;
  }
}

// Offsets of the staged tensors inside the caller's device buffer.
struct Staging {
  size_t k, ks, q, w, idx, val, ws, ws_bytes, total;
};

// rows_per_chunk for T rows: the caller's choice, else about 16 chunks of
// at least 1024 rows; rounded up to a multiple of `align` (4 query rows per
// tensor-core unit, or the group size) and to at most kMaxChunks chunks.
int64_t chunk_rows_for(int64_t T, int64_t chunk_rows, int64_t align) {
  int64_t c = chunk_rows > 0 ? chunk_rows : (T + 15) / 16;
  if (chunk_rows <= 0 && c < 1024) c = 1024;
  const int64_t floor_c = (T + kMaxChunks - 1) / kMaxChunks;
  if (c < floor_c) c = floor_c;
  c = (c + align - 1) / align * align;
  return c < T ? c : T;
}

int prefill_staging(int T, int N, int H, int d, int k, int q_dtype, int k_dtype, size_t ws_bytes, Staging& s) {
  const size_t qe = elem_size(q_dtype), ke = elem_size(k_dtype);
  if (!qe || !ke) return DSA_ERR_INVALID_ARG;
  memset(&s, 0, sizeof(s));
  size_t off = 0;
  s.k = off; off += up256((size_t)N * d * ke);
  s.ks = off; off += k_dtype == DSA_DTYPE_FP8_E4M3 ? up256((size_t)N * 4) : 0;
  s.q = off; off += up256((size_t)T * H * d * qe);
  s.w = off; off += up256((size_t)T * H * 4);
  s.idx = off; off += up256((size_t)T * k * 4);
  s.val = off; off += up256((size_t)T * k * 4);
  s.ws = off; off += up256(ws_bytes);
  s.ws_bytes = ws_bytes;
  s.total = off;
  return DSA_OK;
}

// Streams and events of one call; everything is released by the destructor
// after the streams have drained.
struct Pipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, keys = nullptr, fin = nullptr;
  cudaEvent_t ready[kMaxChunks] = {}, done[kMaxChunks] = {};
  int n = 0;

  int open(int chunks) {
    n = chunks;
    if (cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking) != cudaSuccess) return DSA_ERR_CUDA;
    const unsigned fl = cudaEventDisableTiming;
    if (cudaEventCreateWithFlags(&start, fl) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaEventCreateWithFlags(&keys, fl) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaEventCreateWithFlags(&fin, fl) != cudaSuccess) return DSA_ERR_CUDA;
    for (int c = 0; c < n; ++c) {
      if (cudaEventCreateWithFlags(&ready[c], fl) != cudaSuccess) return DSA_ERR_CUDA;
      if (cudaEventCreateWithFlags(&done[c], fl) != cudaSuccess) return DSA_ERR_CUDA;
    }
    return DSA_OK;
  }

  ~Pipe() {
    if (in) cudaStreamSynchronize(in);
    if (out) cudaStreamSynchronize(out);
    for (int c = 0; c < n; ++c) {
      if (ready[c]) cudaEventDestroy(ready[c]);
      if (done[c]) cudaEventDestroy(done[c]);
    }
    if (start) cudaEventDestroy(start);
    if (keys) cudaEventDestroy(keys);
    if (fin) cudaEventDestroy(fin);
    if (in) cudaStreamDestroy(in);
    if (out) cudaStreamDestroy(out);
  }
};

int h2d(void* dst, const void* src, size_t bytes, cudaStream_t st) {
  if (!bytes) return DSA_OK;
  return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

int d2h(void* dst, const void* src, size_t bytes, cudaStream_t st) {
  if (!bytes) return DSA_OK;
  return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// The chunked prefill pipeline.  `run(r0, n)` launches the indexer on rows
// r0 .. r0+n-1 of the staged tensors on `st`, with the staged workspace.
template <class Run>
int prefill_pipeline(const Staging& s, uint8_t* base, const void* Q, const float* w, const void* K,
                     const float* K_scale, int T, int N, int H, int d, int k, int q_dtype, int k_dtype,
                     int64_t rows_per_chunk, int32_t* idx, float* val, cudaStream_t st, Run run) {
  const size_t qrow = (size_t)H * d * elem_size(q_dtype), wrow = (size_t)H * 4, orow = (size_t)k * 4;
  const int chunks = (int)((T + rows_per_chunk - 1) / rows_per_chunk);
  int r = DSA_OK;
  {
    Pipe p;
    if ((r = p.open(chunks)) != DSA_OK) return r;
    // the staging buffer is the library's: clear its device status word
    if (cudaMemsetAsync(base + s.ws, 0, 8, st) != cudaSuccess) return DSA_ERR_CUDA;
    // the staging buffer may still be read by earlier work on the caller's stream
    if (cudaEventRecord(p.start, st) != cudaSuccess || cudaStreamWaitEvent(p.in, p.start, 0) != cudaSuccess)
      return DSA_ERR_CUDA;
    if ((r = h2d(base + s.k, K, (size_t)N * d * elem_size(k_dtype), p.in)) != DSA_OK) return r;
    if (K_scale && (r = h2d(base + s.ks, K_scale, (size_t)N * 4, p.in)) != DSA_OK) return r;
    if (cudaEventRecord(p.keys, p.in) != cudaSuccess || cudaStreamWaitEvent(st, p.keys, 0) != cudaSuccess)
      return DSA_ERR_CUDA;
    for (int c = 0; c < chunks && r == DSA_OK; ++c) {
      const int64_t r0 = (int64_t)c * rows_per_chunk;
      const int64_t n = T - r0 < rows_per_chunk ? T - r0 : rows_per_chunk;
      if ((r = h2d(base + s.q + r0 * qrow, static_cast<const uint8_t*>(Q) + r0 * qrow, n * qrow, p.in)) != DSA_OK ||
          (r = h2d(base + s.w + r0 * wrow, reinterpret_cast<const uint8_t*>(w) + r0 * wrow, n * wrow, p.in)) != DSA_OK)
        break;
      if (cudaEventRecord(p.ready[c], p.in) != cudaSuccess || cudaStreamWaitEvent(st, p.ready[c], 0) != cudaSuccess) {
        r = DSA_ERR_CUDA;
        break;
      }
      if ((r = run(r0, n)) != DSA_OK) break;
      if (cudaEventRecord(p.done[c], st) != cudaSuccess || cudaStreamWaitEvent(p.out, p.done[c], 0) != cudaSuccess) {
        r = DSA_ERR_CUDA;
        break;
      }
      if ((r = d2h(reinterpret_cast<uint8_t*>(idx) + r0 * orow, base + s.idx + r0 * orow, n * orow, p.out)) != DSA_OK ||
          (r = d2h(reinterpret_cast<uint8_t*>(val) + r0 * orow, base + s.val + r0 * orow, n * orow, p.out)) != DSA_OK)
        break;
    }
    // later work on the caller's stream follows the last copy out
    if (cudaEventRecord(p.fin, p.out) != cudaSuccess || cudaStreamWaitEvent(st, p.fin, 0) != cudaSuccess)
      if (r == DSA_OK) r = DSA_ERR_CUDA;
  }  // Pipe drains both streams here
  const int s2 = dsa_check_status(base + s.ws, st);
  return r != DSA_OK ? r : s2;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

extern "C" {

int dsa_index_dense_host_staging_size(int T, int N, int H, int d, int k, int q_dtype, int k_dtype,
                                      size_t* bytes) {
  if (!bytes) return DSA_ERR_INVALID_ARG;
  size_t ws = 0;
  int r = dsa_index_dense_workspace_size(T, N, H, d, k, q_dtype, k_dtype, &ws);
  if (r != DSA_OK) return r;
  if (T == 0) return (*bytes = ws, DSA_OK);  // empty call: the status word only
  Staging s;
  if ((r = prefill_staging(T, N, H, d, k, q_dtype, k_dtype, ws, s)) != DSA_OK) return r;
  *bytes = s.total;
  return DSA_OK;
}

int dsa_index_dense_host(const void* Q, const float* w, const void* K, const float* K_scale, int T, int N, int H,
                         int d, int64_t q_pos0, int k, int q_dtype, int k_dtype, int chunk_rows, int32_t* idx,
                         float* val, void* staging, size_t staging_bytes, void* stream) {
  if (T == 0)  // no query rows: the device call checks the shape and launches nothing
    return dsa_index_dense(nullptr, nullptr, nullptr, nullptr, 0, N, H, d, q_pos0, k, q_dtype, k_dtype, nullptr,
                           nullptr, nullptr, 0, stream);
  if (!Q || !w || !K || !idx || !val || !staging || !aligned16(staging) || chunk_rows < 0) return DSA_ERR_INVALID_ARG;
  if ((k_dtype == DSA_DTYPE_FP8_E4M3) != (K_scale != nullptr)) return DSA_ERR_INVALID_ARG;
  size_t ws = 0;
  int r = dsa_index_dense_workspace_size(T, N, H, d, k, q_dtype, k_dtype, &ws);
  if (r != DSA_OK) return r;
  if (q_pos0 < 0 || q_pos0 + (int64_t)T > (int64_t)N) return DSA_ERR_INVALID_ARG;
  Staging s;
  if ((r = prefill_staging(T, N, H, d, k, q_dtype, k_dtype, ws, s)) != DSA_OK) return r;
  if (staging_bytes < s.total) return DSA_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(staging);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t qrow = (size_t)H * d * elem_size(q_dtype);
  const int64_t per = chunk_rows_for(T, chunk_rows, 4);
  const float* ks = K_scale ? reinterpret_cast<const float*>(base + s.ks) : nullptr;
  return prefill_pipeline(s, base, Q, w, K, K_scale, T, N, H, d, k, q_dtype, k_dtype, per, idx, val, st,
                          [&](int64_t r0, int64_t n) {
                            return dsa_index_dense(base + s.q + r0 * qrow,
                                                   reinterpret_cast<const float*>(base + s.w) + r0 * H,
                                                   base + s.k, ks, (int)n, N, H, d, q_pos0 + r0, k, q_dtype,
                                                   k_dtype, reinterpret_cast<int32_t*>(base + s.idx) + r0 * k,
                                                   reinterpret_cast<float*>(base + s.val) + r0 * k, base + s.ws,
                                                   s.ws_bytes, st);
                          });
}

int dsa_index_group_host_staging_size(int T, int N, int H, int d, int k, int group, int bank, int q_dtype,
                                      int k_dtype, int chunk_rows, size_t* bytes) {
  if (!bytes || chunk_rows < 0 || group < 1) return DSA_ERR_INVALID_ARG;
  size_t ws = 0;
  const int64_t per = chunk_rows_for(T, chunk_rows, group);
  int r = dsa_index_group_workspace_size((int)per, N, H, d, k, group, bank, q_dtype, k_dtype, &ws);
  if (r != DSA_OK) return r;
  if (T == 0) return (*bytes = ws, DSA_OK);  // empty call: the status word only
  Staging s;
  if ((r = prefill_staging(T, N, H, d, k, q_dtype, k_dtype, ws, s)) != DSA_OK) return r;
  *bytes = s.total;
  return DSA_OK;
}

int dsa_index_group_host(const void* Q, const float* w, const void* K, const float* K_scale, int T, int N, int H,
                         int d, int64_t q_pos0, int k, int group, int bank, int mode, int q_dtype, int k_dtype,
                         int chunk_rows, int32_t* idx, float* val, void* staging, size_t staging_bytes,
                         void* stream) {
  if (T == 0)
    return dsa_index_group(nullptr, nullptr, nullptr, nullptr, 0, N, H, d, q_pos0, k, group, bank, mode, q_dtype,
                           k_dtype, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 0, stream);
  if (!Q || !w || !K || !idx || !val || !staging || !aligned16(staging) || chunk_rows < 0 || group < 1)
    return DSA_ERR_INVALID_ARG;
  if ((k_dtype == DSA_DTYPE_FP8_E4M3) != (K_scale != nullptr)) return DSA_ERR_INVALID_ARG;
  if (q_pos0 < 0 || q_pos0 + (int64_t)T > (int64_t)N) return DSA_ERR_INVALID_ARG;
  size_t need = 0;
  int r = dsa_index_group_host_staging_size(T, N, H, d, k, group, bank, q_dtype, k_dtype, chunk_rows, &need);
  if (r != DSA_OK) return r;
  if (staging_bytes < need) return DSA_ERR_WORKSPACE;
  const int64_t per = chunk_rows_for(T, chunk_rows, group);
  size_t ws = 0;
  if ((r = dsa_index_group_workspace_size((int)per, N, H, d, k, group, bank, q_dtype, k_dtype, &ws)) != DSA_OK)
    return r;
  Staging s;
  if ((r = prefill_staging(T, N, H, d, k, q_dtype, k_dtype, ws, s)) != DSA_OK) return r;
  uint8_t* base = static_cast<uint8_t*>(staging);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t qrow = (size_t)H * d * elem_size(q_dtype);
  const float* ks = K_scale ? reinterpret_cast<const float*>(base + s.ks) : nullptr;
  // chunks start on group boundaries, so every group is whole inside one call
  return prefill_pipeline(s, base, Q, w, K, K_scale, T, N, H, d, k, q_dtype, k_dtype, per, idx, val, st,
                          [&](int64_t r0, int64_t n) {
                            return dsa_index_group(base + s.q + r0 * qrow,
                                                   reinterpret_cast<const float*>(base + s.w) + r0 * H,
                                                   base + s.k, ks, (int)n, N, H, d, q_pos0 + r0, k, group, bank,
                                                   mode, q_dtype, k_dtype,
                                                   reinterpret_cast<int32_t*>(base + s.idx) + r0 * k,
                                                   reinterpret_cast<float*>(base + s.val) + r0 * k, nullptr,
                                                   nullptr, nullptr, nullptr, base + s.ws, s.ws_bytes, st);
                          });
}

int dsa_index_decode_host_staging_size(int B, int total_q, int64_t total_keys, int max_keys, int H, int d, int k,
                                       int q_dtype, int k_dtype, size_t* bytes) {
  if (!bytes || B < 0 || total_q < 0 || total_keys < 0) return DSA_ERR_INVALID_ARG;
  const size_t qe = elem_size(q_dtype), ke = elem_size(k_dtype);
  if (!qe || !ke) return DSA_ERR_INVALID_ARG;
  if (B == 0 && total_keys != 0) return DSA_ERR_INVALID_ARG;
  size_t ws = 0;
  int r = dsa_index_decode_workspace_size(B, total_q, max_keys, H, d, k, q_dtype, k_dtype, &ws);
  if (r != DSA_OK) return r;
  if (B == 0) return (*bytes = ws, DSA_OK);  // empty call: the status word only
  size_t off = 0;
  off += up256((size_t)total_keys * d * ke);                                  // K
  off += k_dtype == DSA_DTYPE_FP8_E4M3 ? up256((size_t)total_keys * 4) : 0;    // K_scale
  off += up256((size_t)total_q * H * d * qe) + up256((size_t)total_q * H * 4);  // Q, w
  off += 2 * up256((size_t)total_q * k * 4);                                  // idx, val
  off += up256((size_t)(B + 1) * 8) + up256((size_t)(B + 1) * 4);             // offsets
  off += up256(ws);
  *bytes = off;
  return DSA_OK;
}

int dsa_index_decode_host(const void* Q, const float* w, const void* K, const float* K_scale,
                          const int64_t* k_offsets, const int32_t* q_offsets, int B, int total_q,
                          int64_t total_keys, int max_keys, int H, int d, int k, int q_dtype, int k_dtype,
                          int32_t* idx, float* val, void* staging, size_t staging_bytes, void* stream) {
  if (B == 0)
    return dsa_index_decode(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 0, total_q, total_keys, max_keys, H,
                            d, k, q_dtype, k_dtype, nullptr, nullptr, nullptr, 0, stream);
  if (!Q || !w || !K || !k_offsets || !q_offsets || !idx || !val || !staging || !aligned16(staging))
    return DSA_ERR_INVALID_ARG;
  if ((k_dtype == DSA_DTYPE_FP8_E4M3) != (K_scale != nullptr)) return DSA_ERR_INVALID_ARG;
  // the offsets are in host memory here: check all of them before anything
  // else (sequence b: 1 <= N_b <= max_keys, 1 <= m_b <= min(4, N_b))
  if (B < 0 || k_offsets[0] != 0 || k_offsets[B] != total_keys || q_offsets[0] != 0 || q_offsets[B] != total_q)
    return DSA_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b) {
    const int64_t nb = k_offsets[b + 1] - k_offsets[b];
    const int64_t mb = (int64_t)q_offsets[b + 1] - q_offsets[b];
    if (nb < 1 || nb > max_keys || mb < 1 || mb > 4 || mb > nb) return DSA_ERR_INVALID_ARG;
  }
  size_t need = 0;
  int r = dsa_index_decode_host_staging_size(B, total_q, total_keys, max_keys, H, d, k, q_dtype, k_dtype, &need);
  if (r != DSA_OK) return r;
  if (staging_bytes < need) return DSA_ERR_WORKSPACE;
  size_t ws = 0;
  if ((r = dsa_index_decode_workspace_size(B, total_q, max_keys, H, d, k, q_dtype, k_dtype, &ws)) != DSA_OK) return r;
  const size_t qe = elem_size(q_dtype), ke = elem_size(k_dtype);
  uint8_t* base = static_cast<uint8_t*>(staging);
  size_t off = 0;
  const size_t o_k = off; off += up256((size_t)total_keys * d * ke);
  const size_t o_ks = off; off += k_dtype == DSA_DTYPE_FP8_E4M3 ? up256((size_t)total_keys * 4) : 0;
  const size_t o_q = off; off += up256((size_t)total_q * H * d * qe);
  const size_t o_w = off; off += up256((size_t)total_q * H * 4);
  const size_t o_idx = off; off += up256((size_t)total_q * k * 4);
  const size_t o_val = off; off += up256((size_t)total_q * k * 4);
  const size_t o_ko = off; off += up256((size_t)(B + 1) * 8);
  const size_t o_qo = off; off += up256((size_t)(B + 1) * 4);
  const size_t o_ws = off;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // decode is one chunk: its key copy dwarfs the scan, so there is nothing
  // to overlap; the copies go on the caller's stream
  const size_t out_bytes = (size_t)total_q * k * 4;
  r = cudaMemsetAsync(base + o_ws, 0, 8, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
  if (r == DSA_OK) r = h2d(base + o_k, K, (size_t)total_keys * d * ke, st);
  if (r == DSA_OK && K_scale) r = h2d(base + o_ks, K_scale, (size_t)total_keys * 4, st);
  if (r == DSA_OK) r = h2d(base + o_q, Q, (size_t)total_q * H * d * qe, st);
  if (r == DSA_OK) r = h2d(base + o_w, w, (size_t)total_q * H * 4, st);
  if (r == DSA_OK) r = h2d(base + o_ko, k_offsets, (size_t)(B + 1) * 8, st);
  if (r == DSA_OK) r = h2d(base + o_qo, q_offsets, (size_t)(B + 1) * 4, st);
  if (r == DSA_OK)
    r = dsa_index_decode(base + o_q, reinterpret_cast<const float*>(base + o_w), base + o_k,
                         K_scale ? reinterpret_cast<const float*>(base + o_ks) : nullptr,
                         reinterpret_cast<const int64_t*>(base + o_ko), reinterpret_cast<const int32_t*>(base + o_qo),
                         B, total_q, total_keys, max_keys, H, d, k, q_dtype, k_dtype,
                         reinterpret_cast<int32_t*>(base + o_idx), reinterpret_cast<float*>(base + o_val),
                         base + o_ws, ws, st);
  if (r == DSA_OK) r = d2h(idx, base + o_idx, out_bytes, st);
  if (r == DSA_OK) r = d2h(val, base + o_val, out_bytes, st);
  // copies already queued read the caller's host buffers: drain them on
  // every path before returning
  if (cudaStreamSynchronize(st) != cudaSuccess && r == DSA_OK) r = DSA_ERR_CUDA;
  const int s2 = dsa_check_status(base + o_ws, st);
  return r != DSA_OK ? r : s2;
}

}  // extern "C"
