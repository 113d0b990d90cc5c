// dsa_aux.cu — the smaller kernels around the score kernels:
//   * proxy_mean: PIVOT proxy per group (mean of the members' q and w);
//   * bank_gather: copies each group's bank keys into a contiguous block so
//     the tensor-core kernel can stream them with TMA tiles;
//   * bank_rank_reuse: ranks each group's bank by (proxy score desc, key
//     asc) with a shared-memory bitonic sort and, for Reuse, hands each
//     member the first k ranked keys it may see;
//   * decode_merge: combines the per-split top-k lists of a decode query.
#include "dsa_common.cuh"
#include "dsa_topk.cuh"
#include "dsa_internal.h"

namespace dsa {

// ---------------------------------------------------------------------------
// proxy: qbar[g] = mean of q over the group's members (fp32 sum, then
// rounded to the input type), wbar[g] = mean of w (fp32).
// ---------------------------------------------------------------------------
// Each thread owns 8 consecutive elements (one 16-byte load per member row
// for bf16 queries), summed over the members in order in fp32.
__global__ void proxy_mean_kernel(const void* __restrict__ Q, const float* __restrict__ w, int T, int H, int d,
                                  int G, int q_dtype, void* __restrict__ qbar, float* __restrict__ wbar) {
  const int g = blockIdx.y;
  const int r0 = g * G, r1 = min(T, r0 + G);
  const float n = (float)(r1 - r0);
  const int64_t hd = (int64_t)H * d;
  const int64_t e0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (e0 < hd) {
    float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (q_dtype == DSA_DTYPE_BF16 && e0 + 8 <= hd) {
      const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(Q);
      for (int r = r0; r < r1; ++r) {
        const uint4 v = *reinterpret_cast<const uint4*>(q + (int64_t)r * hd + e0);
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(p[j]);
          s[2 * j] += f.x;
          s[2 * j + 1] += f.y;
        }
      }
      uint4 o;
      __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
      for (int j = 0; j < 4; ++j) po[j] = __floats2bfloat162_rn(s[2 * j] / n, s[2 * j + 1] / n);
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(qbar) + (int64_t)g * hd + e0) = o;
    } else {
      for (int j = 0; j < 8 && e0 + j < hd; ++j) {
        float a = 0.f;
        for (int r = r0; r < r1; ++r) {
          const int64_t i = (int64_t)r * hd + e0 + j;
          a += (q_dtype == DSA_DTYPE_FP32) ? static_cast<const float*>(Q)[i]
                                           : __bfloat162float(static_cast<const __nv_bfloat16*>(Q)[i]);
        }
        const float m = a / n;
        if (q_dtype == DSA_DTYPE_FP32)
          static_cast<float*>(qbar)[(int64_t)g * hd + e0 + j] = m;
        else
          static_cast<__nv_bfloat16*>(qbar)[(int64_t)g * hd + e0 + j] = __float2bfloat16_rn(m);
      }
    }
  }
  if (blockIdx.x == 0) {
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
      float a = 0.f;
      for (int r = r0; r < r1; ++r) a += w[(int64_t)r * H + h];
      wbar[(int64_t)g * H + h] = a / n;
    }
  }
}

int launch_proxy_mean(const void* Q, const float* w, int T, int H, int d, int G, int q_dtype, void* qbar,
                      float* wbar, cudaStream_t stream) {
  const int ng = (T + G - 1) / G;
  const int64_t chunks = ((int64_t)H * d + 7) / 8;
  const dim3 grid((unsigned)((chunks + 127) / 128), (unsigned)ng);
  proxy_mean_kernel<<<grid, 128, 0, stream>>>(Q, w, T, H, d, G, q_dtype, qbar, wbar);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// bank gather: Kg[g*B + j, :] = K[bank[g*B + j], :] (zero rows for -1).
// Rows are copied 16 bytes per thread.
// ---------------------------------------------------------------------------
__global__ void bank_gather_kernel(const uint4* __restrict__ K, int row_vecs, const int32_t* __restrict__ bank,
                                   int64_t n_rows, uint4* __restrict__ Kg) {
  const int64_t total = n_rows * row_vecs;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / row_vecs;
    const int c = (int)(i - r * row_vecs);
    const int32_t src = bank[r];
    Kg[i] = src >= 0 ? K[(int64_t)src * row_vecs + c] : make_uint4(0u, 0u, 0u, 0u);
  }
}

int launch_bank_gather(const void* K, int k_dtype, int d, const int32_t* bank, int ng, int bank_size, void* Kg,
                       cudaStream_t stream) {
  const int elt = (k_dtype == DSA_DTYPE_FP32) ? 4 : (k_dtype == DSA_DTYPE_BF16 ? 2 : 1);
  const int row_vecs = d * elt / 16;
  bank_gather_kernel<<<148 * 8, 256, 0, stream>>>(static_cast<const uint4*>(K), row_vecs, bank,
                                                   (int64_t)ng * bank_size, static_cast<uint4*>(Kg));
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// bank ranking + Reuse.  One CTA per group; the bank (at most 16384 entries)
// is sorted in shared memory as 64-bit keys (order-preserving score bits,
// inverted key index), largest first.
// ---------------------------------------------------------------------------
constexpr int kRankThreads = 512;

__global__ void __launch_bounds__(kRankThreads) bank_rank_reuse_kernel(int32_t* __restrict__ bank_idx,
                                                                       float* __restrict__ bank_val, int B, int P,
                                                                       int G, int T, int64_t q_pos0, int k,
                                                                       int32_t* __restrict__ out_idx,
                                                                       float* __restrict__ out_val, int do_reuse) {
  extern __shared__ uint64_t keys[];
  const int g = blockIdx.x;
  int32_t* bi = bank_idx + (int64_t)g * B;
  float* bv = bank_val + (int64_t)g * B;
  for (int i = threadIdx.x; i < P; i += blockDim.x) {
    uint64_t key = 0;
    if (i < B && bi[i] >= 0) key = sel_key(make_uint2(__float_as_uint(bv[i]), (uint32_t)bi[i]));
    keys[i] = key;
  }
  __syncthreads();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (P >> 1); i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint64_t x = keys[lo], y = keys[hi];
        if ((x < y) == up) {
          keys[lo] = y;
          keys[hi] = x;
        }
      }
      __syncthreads();
    }
  }
  // ranked bank back to global (empty slots last: -1 / -inf)
  for (int i = threadIdx.x; i < B; i += blockDim.x) {
    const uint64_t key = keys[i];
    if (key == 0) {
      bi[i] = -1;
      bv[i] = __int_as_float(0xff800000);
    } else {
      const uint32_t o = (uint32_t)(key >> 32);
      const uint32_t u = (o & 0x80000000u) ? (o & 0x7fffffffu) : ~o;
      bi[i] = (int32_t)(~(uint32_t)key);
      bv[i] = __uint_as_float(u);
    }
  }
  if (!do_reuse) return;
  __syncthreads();
  // Reuse: warp per member, first k ranked keys with position <= p_t
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int r0 = g * G, r1 = min(T, r0 + G);
  for (int r = r0 + warp; r < r1; r += nw) {
    const int64_t p = q_pos0 + r;
    int32_t* oi = out_idx + (int64_t)r * k;
    float* ov = out_val + (int64_t)r * k;
    int cnt = 0;
    for (int i0 = 0; i0 < B && cnt < k; i0 += 32) {
      const int i = i0 + lane;
      uint64_t key = (i < B) ? keys[i] : 0;
      const int32_t kidx = (int32_t)(~(uint32_t)key);
      const bool keep = key != 0 && (int64_t)kidx <= p;
      const unsigned m = __ballot_sync(0xffffffffu, keep);
      const int rank = cnt + __popc(m & ((1u << lane) - 1u));
      if (keep && rank < k) {
        const uint32_t o = (uint32_t)(key >> 32);
        const uint32_t u = (o & 0x80000000u) ? (o & 0x7fffffffu) : ~o;
        oi[rank] = kidx;
        ov[rank] = __uint_as_float(u);
      }
      cnt += __popc(m);
    }
    for (int i = min(cnt, k) + lane; i < k; i += 32) {
      oi[i] = -1;
      ov[i] = __int_as_float(0xff800000);
    }
  }
}

int launch_bank_rank_reuse(int32_t* bank_idx, float* bank_val, int ng, int bank_size, int G, int T, int64_t q_pos0,
                           int k, int32_t* out_idx, float* out_val, int do_reuse, cudaStream_t stream) {
  int P = 1;
  while (P < bank_size) P <<= 1;
  if (P > 16384) return DSA_ERR_UNSUPPORTED;
  const size_t smem = (size_t)P * sizeof(uint64_t);
  if (smem > 48 * 1024 && cudaFuncSetAttribute(bank_rank_reuse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem) != cudaSuccess)
    return DSA_ERR_CUDA;
  bank_rank_reuse_kernel<<<ng, kRankThreads, smem, stream>>>(bank_idx, bank_val, bank_size, P, G, T, q_pos0, k,
                                                             out_idx, out_val, do_reuse);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// decode merge: per query row, its splits' top-k lists are compacted into one
// contiguous list while their histogram is built (one pass, batched loads),
// the exact threshold bin is read off the histogram, and the row is selected.
// ---------------------------------------------------------------------------
constexpr int kMergeThreads = 256;
constexpr int kMergeStage = 2048;

struct MergeSmem {
  RowState st;
  uint2 stage[kMergeStage];
  int base[257];  // prefix sums of the splits' counts
};

__global__ void __launch_bounds__(kMergeThreads) decode_merge_kernel(const int32_t* __restrict__ part_idx,
                                                                     const float* __restrict__ part_val,
                                                                     const int* __restrict__ part_cnt, int splits,
                                                                     int k, int32_t* __restrict__ out_idx,
                                                                     float* __restrict__ out_val,
                                                                     uint2* __restrict__ scratch, int* status) {
  __shared__ MergeSmem M;
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
  RowState& st = M.st;
  row_reset(st, tid, kMergeThreads);
  if (tid == 0) {
    int acc = 0;
    for (int s = 0; s < splits; ++s) {
      M.base[s] = acc;
      acc += part_cnt[(int64_t)row * splits + s];
    }
    M.base[splits] = acc;
  }
  __syncthreads();
  uint2* cand = scratch + (int64_t)row * splits * k;
  for (int s = 0; s < splits; ++s) {
    const int64_t o = ((int64_t)row * splits + s) * k;
    const int c = M.base[s + 1] - M.base[s], b0 = M.base[s];
    for (int i0 = 0; i0 < c; i0 += kMergeThreads * 4) {
      uint2 e[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = i0 + j * kMergeThreads + tid;
        e[j] = (i < c) ? make_uint2(__float_as_uint(part_val[o + i]), (uint32_t)part_idx[o + i]) : make_uint2(0, 0);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = i0 + j * kMergeThreads + tid;
        if (i < c) {
          cand[b0 + i] = e[j];
          atomicAdd(&st.hist[score_bin(__uint_as_float(e[j].x))], 1u);
        }
      }
    }
  }
  __syncthreads();
  if (tid < 32) {
    const int2 r = hist_scan(st, 0, kBins - 1, k, lane);
    if (lane == 0) {
      st.bstar = r.x >= 0 ? r.x : 0;
      st.cge = r.y;
    }
  }
  __syncthreads();
  row_select(st, single_list(cand, &M.base[splits]), k, row_out(out_idx + (int64_t)row * k, out_val + (int64_t)row * k),
             M.stage, kMergeStage, tid, kMergeThreads, 1, status);
}

int launch_decode_merge(const int32_t* part_idx, const float* part_val, const int* part_cnt, int total_q,
                        int splits, int k, int32_t* out_idx, float* out_val, uint2* scratch, int* status,
                        cudaStream_t stream) {
  if (splits > 256) return DSA_ERR_UNSUPPORTED;
  decode_merge_kernel<<<total_q, kMergeThreads, 0, stream>>>(part_idx, part_val, part_cnt, splits, k, out_idx,
                                                              out_val, scratch, status);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// fp8 e4m3 keys -> bf16 (every e4m3 value is exactly a bf16 value), 16 keys'
// bytes per thread per step.
// ---------------------------------------------------------------------------
__global__ void e4m3_to_bf16_kernel(const uint4* __restrict__ src, int64_t n16, uint4* __restrict__ dst) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n16; i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = src[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float a = e4m3_to_f32((uint8_t)(w[j] >> (16 * h)));
        const float b = e4m3_to_f32((uint8_t)(w[j] >> (16 * h + 8)));
        const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
        o[2 * j + h] = *reinterpret_cast<const uint32_t*>(&p);
      }
    }
    dst[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

int launch_e4m3_to_bf16(const uint8_t* src, int64_t n, void* dst, cudaStream_t stream) {
  e4m3_to_bf16_kernel<<<148 * 8, 256, 0, stream>>>(reinterpret_cast<const uint4*>(src), n / 16,
                                                    static_cast<uint4*>(dst));
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
__global__ void fill_neg_inf_kernel(float* S, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    S[i] = __int_as_float(0xff800000);
}

int launch_fill_scores(float* S, int64_t n, cudaStream_t stream) {
  fill_neg_inf_kernel<<<592, 256, 0, stream>>>(S, n);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
