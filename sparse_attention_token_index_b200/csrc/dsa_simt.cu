// dsa_simt.cu — exact fp32 CUDA-core lightning-indexer kernel.
//
// Serves fp32 inputs (where tf32 tensor-core rounding would not hold the
// scores to 1e-3 under cancellation) and shapes outside the tensor-core
// kernel's H = 64, d = 128 (bf16 q, fp8 or bf16 keys).  Each 128-thread group
// follows one query row: thread i scores key (tile * 128 + i) with fp32 FMAs
// on q staged in shared memory, then the same streaming top-k as the
// tensor-core kernel filters and finally selects.
#include "dsa_common.cuh"
#include "dsa_topk.cuh"
#include "dsa_internal.h"

namespace dsa {

constexpr int kSimtThreads = 256;  // two groups of 128
constexpr int kSimtStageCap = 1024;

__device__ __forceinline__ float load_q(const void* Q, int dt, int64_t i) {
  if (dt == DSA_DTYPE_FP32) return static_cast<const float*>(Q)[i];
  return __bfloat162float(static_cast<const __nv_bfloat16*>(Q)[i]);
}

__device__ __forceinline__ float load_k(const void* K, int dt, int64_t i) {
  if (dt == DSA_DTYPE_FP32) return static_cast<const float*>(K)[i];
  if (dt == DSA_DTYPE_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(K)[i]);
  return e4m3_to_f32(static_cast<const uint8_t*>(K)[i]);
}

struct SimtGroupSmem {
  RowState st;
  uint2 stage[kSimtStageCap];
};

static __host__ __device__ __forceinline__ size_t simt_group_bytes(int H, int d) {
  return (sizeof(SimtGroupSmem) + sizeof(float) * ((size_t)H * d + H) + 15) & ~(size_t)15;
}

size_t simt_smem_bytes(int H, int d) { return 2 * simt_group_bytes(H, d); }

__global__ void __launch_bounds__(kSimtThreads) simt_index_kernel(const SimtArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int wg = threadIdx.x >> 7, tid = threadIdx.x & 127, lane = threadIdx.x & 31, lw = tid >> 5;
  const int bar = 1 + wg;
  const size_t gbytes = simt_group_bytes(a.H, a.d);
  uint8_t* base = smem_raw + wg * gbytes;
  SimtGroupSmem& G = *reinterpret_cast<SimtGroupSmem*>(base);
  float* qs = reinterpret_cast<float*>(base + sizeof(SimtGroupSmem));
  float* ws = qs + (size_t)a.H * a.d;
  const int H = a.H, d = a.d;

  for (int task = blockIdx.x * 2 + wg; task < a.n_tasks; task += gridDim.x * 2) {
    int64_t row, pos, key_row0;
    int key_begin, key_end;  // local key range scanned
    int64_t out_row;
    if (a.kind == 0) {
      row = task;
      pos = a.q_pos0 + row;
      key_row0 = 0;
      key_begin = 0;
      key_end = (int)(pos + 1);
      out_row = row;
    } else {
      const int qrow = task / a.splits, sp = task % a.splits;
      int b = 0;
      while (b < a.B && a.q_off[b + 1] <= qrow) ++b;
      const int64_t k0 = b < a.B ? a.k_off[b] : 0, k1 = b < a.B ? a.k_off[b + 1] : 0;
      const int q0 = b < a.B ? a.q_off[b] : 0;
      const int mb = b < a.B ? a.q_off[b + 1] - q0 : 0;
      // the row's sequence must exist, lie inside K, fit this plan's slices
      // (N_b <= max_keys) and have 1 <= m_b <= min(4, N_b): otherwise its
      // partial lists stay empty and the call reports an invalid argument
      if (b >= a.B || k0 < 0 || k1 - k0 < 1 || k1 > a.total_keys || k1 - k0 > (int64_t)a.splits * a.keys_per_split ||
          q0 < 0 || qrow < q0 || mb < 1 || mb > 4 || (int64_t)mb > k1 - k0) {
        if (tid == 0) {
          report_error(a.status, DSA_ERR_INVALID_ARG, 7);
          a.out_cnt[(int64_t)qrow * a.splits + sp] = 0;
        }
        continue;
      }
      const int j = qrow - q0;
      const int nb = (int)(k1 - k0);
      row = qrow;
      pos = (int64_t)nb - mb + j;
      key_row0 = k0;
      key_begin = min(nb, sp * a.keys_per_split);
      key_end = min((int)(pos + 1), min(nb, key_begin + a.keys_per_split));
      if (key_end < key_begin) key_end = key_begin;
      out_row = (int64_t)qrow * a.splits + sp;
    }
    for (int i = tid; i < H * d; i += 128) qs[i] = load_q(a.Q, a.q_dtype, row * H * d + i);
    for (int i = tid; i < H; i += 128) ws[i] = a.w[row * H + i];
    row_reset(G.st, tid, 128);
    uint2* cand = a.cand + ((int64_t)blockIdx.x * 2 + wg) * a.cand_cap;
    named_bar(bar, 128);
    for (int t0 = key_begin; t0 < key_end; t0 += 128) {
      const int key = t0 + tid;
      const bool valid = key < key_end;
      float score = 0.f;
      if (valid) {
        const int64_t kr = (key_row0 + key) * (int64_t)d;
        for (int h = 0; h < H; ++h) {
          float dot = 0.f;
          for (int i = 0; i < d; ++i) dot = fmaf(qs[h * d + i], load_k(a.K, a.k_dtype, kr + i), dot);
          score = fmaf(ws[h], fmaxf(dot, 0.f), score);
        }
        if (a.k_dtype == DSA_DTYPE_FP8_E4M3) score *= a.K_scale[key_row0 + key];
        score = score + 0.0f;
        if (a.dbg_scores != nullptr) a.dbg_scores[row * a.dbg_ld + key] = score;
      }
      row_append(G.st, cand, score, (uint32_t)key, valid, lane, a.cand_cap, a.status);
      named_bar(bar, 128);
      if (lw == 0) row_update(G.st, a.k, lane);
      named_bar(bar, 128);
    }
    const RowOut out = a.kind == 1 ? pair_out(a.out_pair + out_row * a.out_ld, a.k, a.status)
                                   : row_out(a.out_idx + out_row * a.out_ld, a.out_val + out_row * a.out_ld, a.k,
                                             a.status);
    const int cnt =
        row_select(G.st, single_list(cand, &G.st.cnt), a.k, out, G.stage, kSimtStageCap, tid, 128, bar, a.status);
    if (a.kind == 1 && tid == 0) a.out_cnt[out_row] = cnt;
    named_bar(bar, 128);
  }
}

int launch_simt_index(const SimtArgs& a, int grid, cudaStream_t stream) {
  const NvtxRange nvtx(a.kind == 1 ? "dsa.score_topk.decode.fp32" : "dsa.score_topk.fp32");
  const size_t smem = simt_smem_bytes(a.H, a.d);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(simt_index_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
  }
  const TimerSlot ts = timer_acquire();
  if (ts.start) cudaEventRecord(ts.start, stream);
  simt_index_kernel<<<grid, kSimtThreads, smem, stream>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (ts.end) cudaEventRecord(ts.end, stream);
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
