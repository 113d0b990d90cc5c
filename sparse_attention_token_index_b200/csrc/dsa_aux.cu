// dsa_aux.cu — the smaller kernels around the score kernels:
//   * proxy_mean: PIVOT proxy per group (mean of the members' q and w);
//   * bank_gather: copies each group's bank keys into a contiguous block so
//     the tensor-core kernel can stream them with TMA tiles;
//   * bank_rank_reuse: ranks each group's bank by (proxy score desc, key
//     asc) with a shared-memory bitonic sort and, for Reuse, hands each
//     member the first k ranked keys it may see;
//   * decode_merge: combines the per-split top-k lists of a decode query;
//   * local_extend: bank + a group's own stretch (Refine with local additions);
//   * block_mean: block representatives for block routing.
#include <atomic>

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
// Group g is rows gG .. min(T, (g+1)G) - 1, or seg[g] .. seg[g+1] - 1 when
// seg (per-group row offsets, e.g. a decode batch's query offsets) is given.
__global__ void proxy_mean_kernel(const void* __restrict__ Q, const float* __restrict__ w, int T, int H, int d,
                                  int G, const int32_t* __restrict__ seg, int q_dtype, void* __restrict__ qbar,
                                  float* __restrict__ wbar, const int* ok) {
  if (offsets_bad(ok)) return;
  const int g = blockIdx.y;
  const int r0 = seg ? seg[g] : g * G, r1 = seg ? seg[g + 1] : min(T, r0 + G);
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
                      float* wbar, cudaStream_t stream, const int32_t* seg, int nseg, const int* ok) {
  const NvtxRange nvtx("dsa.proxy_mean");
  const int ng = seg ? nseg : (T + G - 1) / G;
  const int64_t chunks = ((int64_t)H * d + 7) / 8;
  const dim3 grid((unsigned)((chunks + 127) / 128), (unsigned)ng);
  proxy_mean_kernel<<<grid, 128, 0, stream>>>(Q, w, T, H, d, G, seg, q_dtype, qbar, wbar, ok);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// block representatives: R[b] = mean of keys b*128 .. min(N, b*128+128) - 1
// (keys times their per-key scale when given), fp32 sums in key order,
// rounded to bf16.  One CTA per block, thread j owns element j.
// ---------------------------------------------------------------------------
__global__ void block_mean_kernel(const __nv_bfloat16* __restrict__ K, const float* __restrict__ K_scale, int64_t N,
                                  int d, __nv_bfloat16* __restrict__ R) {
  const int64_t b = blockIdx.x;
  const int64_t r0 = b * 128, r1 = min(N, r0 + 128);
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float s = 0.f;
    for (int64_t r = r0; r < r1; ++r) {
      const float x = __bfloat162float(K[r * d + j]);
      s += K_scale ? x * K_scale[r] : x;
    }
    R[b * d + j] = __float2bfloat16_rn(s / (float)(r1 - r0));
  }
}

int launch_block_mean(const void* K, const float* K_scale, int64_t N, int d, void* R, cudaStream_t stream) {
  const NvtxRange nvtx("dsa.block_mean");
  const int64_t nb = (N + 127) / 128;
  block_mean_kernel<<<(unsigned)nb, 128, 0, stream>>>(static_cast<const __nv_bfloat16*>(K), K_scale, N, d,
                                                      static_cast<__nv_bfloat16*>(R));
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// bank gather: Kg[g*B + j, :] = K[base_g + bank[g*B + j], :] (zero rows for
// -1), base_g = row_off[g] when the bank holds indices local to a sequence
// (decode), else 0.  Rows are copied 16 bytes per thread.
// ---------------------------------------------------------------------------
__global__ void bank_gather_kernel(const uint4* __restrict__ K, int row_vecs, const int32_t* __restrict__ bank,
                                   int64_t n_rows, int bank_size, const int64_t* __restrict__ row_off,
                                   uint4* __restrict__ Kg, const int* ok) {
  if (offsets_bad(ok)) return;
  const int64_t total = n_rows * row_vecs;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / row_vecs;
    const int c = (int)(i - r * row_vecs);
    const int32_t src = bank[r];
    const int64_t base = row_off ? row_off[r / bank_size] : 0;
    Kg[i] = src >= 0 ? K[(base + src) * row_vecs + c] : make_uint4(0u, 0u, 0u, 0u);
  }
}

// The tensor-core path's rows (bf16, d = 128: 16 vectors of 16 bytes): a warp
// copies two whole rows per step, one bank entry read per row and no
// division per element, so the copy runs at the write bandwidth.
__global__ void bank_gather_rows16_kernel(const uint4* __restrict__ K, const int32_t* __restrict__ bank,
                                          int64_t n_rows, int bank_size, const int64_t* __restrict__ row_off,
                                          uint4* __restrict__ Kg, const int* ok) {
  if (offsets_bad(ok)) return;
  const int lane = threadIdx.x & 31, c = lane & 15;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t r = warp0 * 2 + (lane >> 4); r < n_rows; r += nwarps * 2) {
    const int32_t src = bank[r];
    const int64_t base = row_off ? row_off[r / bank_size] : 0;
    Kg[r * 16 + c] = src >= 0 ? K[(base + src) * 16 + c] : make_uint4(0u, 0u, 0u, 0u);
  }
}

// Refine's bank in descending order of the proxy's score bin, then gathered:
// map[g, :] = the group's bank indices ordered by score_bin(proxy score),
// highest bin first (any order inside a bin), and Kg the matching key rows
// (bf16, d = 128).  Members then meet their likely top keys early, so their
// streaming threshold rises sooner and fewer candidates reach the select.
// The bank stays the same set: the order changes nothing in the results.
// One block of kOrderThreads per group.
constexpr int kOrderThreads = 512;
constexpr int kOrderMaxBank = 8192;  // bank entries a block orders in shared memory

__global__ void __launch_bounds__(kOrderThreads) bank_order_gather_kernel(const uint4* __restrict__ K,
                                                                           const int32_t* __restrict__ bank_idx,
                                                                           const float* __restrict__ bank_val,
                                                                           int bank_size, int32_t* __restrict__ map,
                                                                           uint4* __restrict__ Kg) {
  __shared__ int hist[kBins];
  __shared__ int32_t smap[kOrderMaxBank];
  const int g = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t* bi = bank_idx + (int64_t)g * bank_size;
  const float* bv = bank_val + (int64_t)g * bank_size;
  for (int b = tid; b < kBins; b += kOrderThreads) hist[b] = 0;
  __syncthreads();
  for (int j = tid; j < bank_size; j += kOrderThreads) atomicAdd(&hist[score_bin(bv[j])], 1);
  __syncthreads();
  if (warp == 0) {
    // start of each bin in descending bin order: lane l owns bins 1023 - 32l - 31 .. 1023 - 32l
    int c[32];
    int tot = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      c[i] = hist[kBins - 1 - 32 * lane - i];
      tot += c[i];
    }
    int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - tot;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      hist[kBins - 1 - 32 * lane - i] = run;  // becomes the bin's next free slot
      run += c[i];
    }
  }
  __syncthreads();
  for (int j = tid; j < bank_size; j += kOrderThreads) smap[atomicAdd(&hist[score_bin(bv[j])], 1)] = bi[j];
  __syncthreads();
  int32_t* mg = map + (int64_t)g * bank_size;
  for (int j = tid; j < bank_size; j += kOrderThreads) mg[j] = smap[j];
  // the key rows, two 256-byte rows a warp step
  const int c16 = lane & 15;
  uint4* kg = Kg + (int64_t)g * bank_size * 16;
  for (int r = warp * 2 + (lane >> 4); r < bank_size; r += (kOrderThreads / 32) * 2) {
    const int32_t src = smap[r];
    kg[(int64_t)r * 16 + c16] = src >= 0 ? K[(int64_t)src * 16 + c16] : make_uint4(0u, 0u, 0u, 0u);
  }
}

int launch_bank_order_gather(const void* K, const int32_t* bank_idx, const float* bank_val, int ng, int bank_size,
                             int32_t* map, void* Kg, cudaStream_t stream) {
  const NvtxRange nvtx("dsa.bank_order_gather");
  if (bank_size > kOrderMaxBank) return DSA_ERR_UNSUPPORTED;
  if (ng == 0) return DSA_OK;
  bank_order_gather_kernel<<<ng, kOrderThreads, 0, stream>>>(static_cast<const uint4*>(K), bank_idx, bank_val,
                                                             bank_size, map, static_cast<uint4*>(Kg));
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

int launch_bank_gather(const void* K, int k_dtype, int d, const int32_t* bank, int ng, int bank_size, void* Kg,
                       cudaStream_t stream, const int64_t* row_off, const int* ok) {
  const NvtxRange nvtx("dsa.bank_gather");
  const int elt = (k_dtype == DSA_DTYPE_FP32) ? 4 : (k_dtype == DSA_DTYPE_BF16 ? 2 : 1);
  const int row_vecs = d * elt / 16;
  if (row_vecs == 16)
    bank_gather_rows16_kernel<<<148 * 8, 256, 0, stream>>>(static_cast<const uint4*>(K), bank,
                                                           (int64_t)ng * bank_size, bank_size, row_off,
                                                           static_cast<uint4*>(Kg), ok);
  else
    bank_gather_kernel<<<148 * 8, 256, 0, stream>>>(static_cast<const uint4*>(K), row_vecs, bank,
                                                     (int64_t)ng * bank_size, bank_size, row_off,
                                                     static_cast<uint4*>(Kg), ok);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Refine with query-specific additions: map[g] = the group's bank (B slots),
// then S - B slots for its own stretch of positions p_first .. p_first + m - 1
// (m members; -1 beyond), each -1 when the bank holds that key already, so
// that no key is a candidate twice.  Decode groups (q_off / k_off): sequence
// g, p_first = N_g - m_g, local indices.
// ---------------------------------------------------------------------------
__global__ void local_extend_kernel(const int32_t* __restrict__ bank, int B, int G, int T, int64_t q_pos0,
                                    const int32_t* __restrict__ q_off, const int64_t* __restrict__ k_off, int S,
                                    int32_t* __restrict__ map, const int* ok) {
  extern __shared__ int in_bank[];  // [S - B]
  if (offsets_bad(ok)) return;
  const int g = blockIdx.x, tid = threadIdx.x;
  const int W = S - B;
  int r0, r1;
  int64_t p_first;
  if (q_off) {
    r0 = q_off[g];
    r1 = q_off[g + 1];
    p_first = (k_off[g + 1] - k_off[g]) - (r1 - r0);
  } else {
    r0 = g * G;
    r1 = min(T, r0 + G);
    p_first = q_pos0 + r0;
  }
  const int m = r1 - r0;
  for (int i = tid; i < W; i += blockDim.x) in_bank[i] = 0;
  __syncthreads();
  for (int j = tid; j < B; j += blockDim.x) {
    const int32_t key = bank[(int64_t)g * B + j];
    map[(int64_t)g * S + j] = key;
    const int64_t o = (int64_t)key - p_first;
    if (key >= 0 && o >= 0 && o < m) in_bank[o] = 1;
  }
  __syncthreads();
  for (int i = tid; i < W; i += blockDim.x)
    map[(int64_t)g * S + B + i] = (i < m && !in_bank[i]) ? (int32_t)(p_first + i) : -1;
}

int launch_local_extend(const int32_t* bank, int ng, int B, int G, int T, int64_t q_pos0, const int32_t* q_off,
                        const int64_t* k_off, int S, int32_t* map, cudaStream_t stream, const int* ok) {
  const NvtxRange nvtx("dsa.local_extend");
  if (S - B < 1 || S - B > 4096) return DSA_ERR_INVALID_ARG;
  local_extend_kernel<<<ng, 256, (size_t)(S - B) * sizeof(int), stream>>>(bank, B, G, T, q_pos0, q_off, k_off, S,
                                                                          map, ok);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// bank ranking + Reuse.  One CTA per group; the bank (at most 16384 entries)
// is held in shared memory as 64-bit keys (order-preserving score bits,
// inverted key index: larger key = higher rank, unique per entry).
//   M == B: the whole bank is sorted, largest first, and written back.
//   M <  B: only the M highest keys are needed (Reuse without a bank output:
//           member t drops at most G - 1 bank keys, those of its own group
//           above p_t, so its first k lie among the top k + G - 1).  An MSD
//           radix select on 8-bit digits finds the M-th key, the M keys at or
//           above it are compacted and only they are sorted.
// ---------------------------------------------------------------------------
constexpr int kRankThreads = 512;

__global__ void __launch_bounds__(kRankThreads) bank_rank_reuse_kernel(int32_t* __restrict__ bank_idx,
                                                                       float* __restrict__ bank_val, int B, int P,
                                                                       int M, int PM, int G, int T, int64_t q_pos0,
                                                                       int k, int32_t* __restrict__ out_idx,
                                                                       float* __restrict__ out_val, int do_reuse,
                                                                       const int32_t* __restrict__ q_off,
                                                                       const int64_t* __restrict__ k_off,
                                                                       const int* ok) {
  extern __shared__ uint64_t keys[];  // [P] the bank; then [PM] its top M when M < B
  __shared__ uint32_t hist[256];
  __shared__ int sh_digit, sh_above, sh_in, sh_cnt;
  if (offsets_bad(ok)) return;
  const int g = blockIdx.x, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  int32_t* bi = bank_idx + (int64_t)g * B;
  float* bv = bank_val + (int64_t)g * B;
  if (tid == 0) sh_cnt = 0;
  int mine = 0;
  for (int i = tid; i < P; i += blockDim.x) {
    uint64_t key = 0;
    if (i < B && bi[i] >= 0) key = sel_key(make_uint2(__float_as_uint(bv[i]), (uint32_t)bi[i]));
    keys[i] = key;
    mine += key != 0;
  }
  __syncthreads();
  if (mine) atomicAdd(&sh_cnt, mine);
  __syncthreads();
  const int nvalid = sh_cnt;
  __syncthreads();  // every thread has read the count before sh_cnt is reused
  uint64_t* rk = keys;  // the array that gets sorted, R entries
  int R = P;
  if (M < B) {
    uint64_t prefix = 0, mask = 0;
    if (nvalid > M) {
      int remaining = M;
      for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < P; i += blockDim.x) {
          const uint64_t key = keys[i];
          if (key != 0 && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (warp == 0) {
          // digit holding the remaining-th largest, scanning from digit 255 down
          uint32_t c[8], tot = 0;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            c[j] = hist[255 - 8 * lane - j];
            tot += c[j];
          }
          uint32_t incl = tot;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          const uint32_t excl = incl - tot;
          if (excl < (uint32_t)remaining && incl >= (uint32_t)remaining) {
            uint32_t cum = excl;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              if (cum + c[j] >= (uint32_t)remaining) {
                sh_digit = 255 - 8 * lane - j;
                sh_above = (int)cum;
                sh_in = (int)c[j];
                break;
              }
              cum += c[j];
            }
          }
        }
        __syncthreads();
        const int dsel = sh_digit, above = sh_above, in = sh_in;
        __syncthreads();
        remaining -= above;
        prefix |= (uint64_t)dsel << shift;
        mask |= (uint64_t)0xFFu << shift;
        // keys with (key & mask) >= prefix: the M - remaining already above
        // this bucket plus the bucket itself.  Once they fit the sort buffer
        // the digit steps can stop: the sort ranks the surplus below the top
        // M, and members read the first M ranks only.
        if (M - remaining + in <= PM) break;
      }
    }
    // compact the keys at or above the prefix (at most PM, the top M among
    // them; any order), then sort only them
    uint64_t* top = keys + P;
    if (tid == 0) sh_cnt = 0;
    __syncthreads();
    for (int i = tid; i < P; i += blockDim.x) {
      const uint64_t key = keys[i];
      if (key != 0 && (key & mask) >= prefix) top[atomicAdd(&sh_cnt, 1)] = key;
    }
    __syncthreads();
    for (int i = sh_cnt + tid; i < PM; i += blockDim.x) top[i] = 0;
    __syncthreads();
    rk = top;
    R = PM;
  }
  for (int size = 2; size <= R; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < (R >> 1); i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint64_t x = rk[lo], y = rk[hi];
        if ((x < y) == up) {
          rk[lo] = y;
          rk[hi] = x;
        }
      }
      __syncthreads();
    }
  }
  if (M == B) {
    // ranked bank back to global (empty slots last: -1 / -inf)
    for (int i = tid; i < B; i += blockDim.x) {
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
  }
  if (!do_reuse) return;
  const int NR = M < R ? M : R;  // ranked entries a member may take from
  // Reuse: warp per member, first k ranked keys with position <= p_t.  A
  // decode group (q_off / k_off given) is sequence g: members q_off[g] ..
  // q_off[g+1] - 1, member j at N_g - m_g + j with local key indices.
  const int r0 = q_off ? q_off[g] : g * G, r1 = q_off ? q_off[g + 1] : min(T, r0 + G);
  const int64_t p0 = q_off ? (k_off[g + 1] - k_off[g]) - (r1 - r0) - r0 : q_pos0;
  for (int r = r0 + warp; r < r1; r += nw) {
    const int64_t p = p0 + r;
    int32_t* oi = out_idx + (int64_t)r * k;
    float* ov = out_val + (int64_t)r * k;
    int cnt = 0;
    for (int i0 = 0; i0 < NR && cnt < k; i0 += 32) {
      const int i = i0 + lane;
      uint64_t key = (i < NR) ? rk[i] : 0;
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
                           int k, int32_t* out_idx, float* out_val, int do_reuse, int rank_all, cudaStream_t stream,
                           const int32_t* q_off, const int64_t* k_off, const int* ok) {
  const NvtxRange nvtx("dsa.bank_rank_reuse");
  int P = 1;
  while (P < bank_size) P <<= 1;
  if (P > kMaxBank) return DSA_ERR_UNSUPPORTED;
  int M = bank_size, PM = 0;
  if (!rank_all) {
    const int64_t m = (int64_t)k + G - 1;
    if (m < bank_size) {
      PM = 1;
      while (PM < m) PM <<= 1;
      if ((size_t)(P + PM) * sizeof(uint64_t) <= 200 * 1024) M = (int)m;
      else PM = 0;
    }
  }
  const size_t smem = (size_t)(P + PM) * sizeof(uint64_t);
  if (smem > 48 * 1024 && cudaFuncSetAttribute(bank_rank_reuse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem) != cudaSuccess)
    return DSA_ERR_CUDA;
  bank_rank_reuse_kernel<<<ng, kRankThreads, smem, stream>>>(bank_idx, bank_val, bank_size, P, M, PM, G, T, q_pos0, k,
                                                             out_idx, out_val, do_reuse, q_off, k_off, ok);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// decode merge: per query row, its splits' top-k lists (packed pairs) are one
// segmented candidate list.  One pass builds their histogram, the exact
// threshold bin is read off it, and the row is selected straight from the
// lists (no copy).
// ---------------------------------------------------------------------------
constexpr int kMergeThreads = 512;
constexpr int kMergeStage = 4096;  // <= 8 entries per thread for the stage resolve

struct MergeSmem {
  RowState st;
  uint2 stage[kMergeStage];
};

__global__ void __launch_bounds__(kMergeThreads) decode_merge_kernel(const uint2* __restrict__ parts,
                                                                     const int* __restrict__ part_cnt, int splits,
                                                                     int k, int32_t* __restrict__ out_idx,
                                                                     float* __restrict__ out_val, int* status,
                                                                     const int* ok) {
  __shared__ MergeSmem M;
  __shared__ int cnt[256];
  if (offsets_bad(ok)) return;
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
  RowState& st = M.st;
  row_reset(st, tid, kMergeThreads);
  // a split holds at most k entries; a count outside [0, k] (a slice the scan
  // skipped because its sequence's offsets were invalid) reads as empty
  for (int s = tid; s < splits; s += kMergeThreads) {
    const int c = __ldcg(part_cnt + (int64_t)row * splits + s);
    cnt[s] = (c >= 0 && c <= k) ? c : 0;
  }
  CandList cl;
  cl.base = parts + (int64_t)row * splits * k;
  cl.stride = k;
  cl.nseg = splits;
  cl.cnt = cnt;
  cl.l2 = true;  // written by the scoring kernel's other CTAs
  __syncthreads();
  for_each_cand(cl, tid, kMergeThreads, [&](uint2 e, bool v) {
    if (v) atomicAdd(&st.hist[score_bin(__uint_as_float(e.x))], 1u);
  });
  __syncthreads();
  if (tid < 32) {
    const int2 r = hist_scan(st, 0, kBins - 1, k, lane);
    if (lane == 0) {
      st.bstar = r.x >= 0 ? r.x : 0;
      st.cge = r.y;
    }
  }
  __syncthreads();
  row_select(st, cl, k, row_out(out_idx + (int64_t)row * k, out_val + (int64_t)row * k, k, status), M.stage,
             kMergeStage, tid, kMergeThreads, 1, status);
}

int launch_decode_merge(const uint2* parts, const int* part_cnt, int total_q, int splits, int k, int32_t* out_idx,
                        float* out_val, int* status, cudaStream_t stream, const int* ok) {
  const NvtxRange nvtx("dsa.decode_merge");
  if (splits > 256) return DSA_ERR_UNSUPPORTED;
  decode_merge_kernel<<<total_q, kMergeThreads, 0, stream>>>(parts, part_cnt, splits, k, out_idx, out_val, status,
                                                             ok);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// decode merge of the tensor-core scan's raw slice lists: a decode row's
// slices left their whole candidate lists (no per-slice selection) with a bin
// histogram each.  The histograms add up to the row's, whose exact threshold
// bin is read off it; one classify pass over every slice's segments (dealt
// out to the warps) emits the entries above it and stages the bin, which the
// same exact resolve as the scan kernel's select finishes.
// ---------------------------------------------------------------------------
constexpr int kMergeListThreads = 1024;

__global__ void __launch_bounds__(kMergeListThreads) decode_merge_lists_kernel(
    const uint2* __restrict__ cand, int64_t cand_cap, const int* __restrict__ hdr, const uint32_t* __restrict__ hist,
    int splits, int k, int32_t* __restrict__ out_idx, float* __restrict__ out_val, int* status, const int* ok) {
  __shared__ MergeSmem M;
  extern __shared__ uint8_t dyn[];  // [splits * 16] segment starts, then [splits * 16] counts
  if (offsets_bad(ok)) return;
  const uint2** segp = reinterpret_cast<const uint2**>(dyn);
  int* segn = reinterpret_cast<int*>(dyn + sizeof(const uint2*) * splits * 16);
  __shared__ int row_nseg;
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
  RowState& st = M.st;
  if (tid == 0) {
    st.outpos = 0;
    st.stage_cnt = 0;
    // a row's slices come from one sequence and share its segment count
    const int ns = __ldcg(hdr + (int64_t)row * splits * kSegHdr);
    row_nseg = (ns == 4 || ns == 8 || ns == 16) ? ns : 0;
  }
  // the row's histogram: the sum of its slices' (loads in flight together)
  for (int b = tid; b < kBins; b += kMergeListThreads) {
    const uint32_t* hb = hist + (int64_t)row * splits * kBins + b;
    uint32_t h0 = 0, h1 = 0, h2 = 0, h3 = 0;
    int sp = 0;
    for (; sp + 4 <= splits; sp += 4) {
      h0 += __ldcg(hb + (int64_t)(sp + 0) * kBins);
      h1 += __ldcg(hb + (int64_t)(sp + 1) * kBins);
      h2 += __ldcg(hb + (int64_t)(sp + 2) * kBins);
      h3 += __ldcg(hb + (int64_t)(sp + 3) * kBins);
    }
    for (; sp < splits; ++sp) h0 += __ldcg(hb + (int64_t)sp * kBins);
    st.hist[b] = (h0 + h1) + (h2 + h3);
  }
  __syncthreads();
  // the segment table, segment j of slice sp at s = j * splits + sp; a slice
  // whose header disagrees (skipped on invalid offsets) reads as empty
  const int ns = row_nseg;
  const int nseg_total = ns * splits;
  const int64_t stride = ns ? cand_cap / ns : 0;
  for (int s = tid; s < nseg_total; s += kMergeListThreads) {
    const int j = s / splits, sp = s - j * splits;
    const int64_t o = (int64_t)row * splits + sp;
    const int c = __ldcg(hdr + o * kSegHdr + 1 + j);
    const bool same = __ldcg(hdr + o * kSegHdr) == ns;
    segp[s] = cand + o * cand_cap + j * stride;
    segn[s] = (same && c >= 0 && c <= stride) ? c : 0;
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
  CandList cl;
  cl.base = cand;
  cl.stride = 0;
  cl.nseg = nseg_total;
  cl.cnt = segn;
  cl.l2 = true;  // written by the scan kernel's CTAs
  cl.segp = segp;
  row_select(st, cl, k, row_out(out_idx + (int64_t)row * k, out_val + (int64_t)row * k, k, status), M.stage,
             kMergeStage, tid, kMergeListThreads, 1, status);
}

int launch_decode_merge_lists(const uint2* cand, int64_t cand_cap, const int* hdr, const uint32_t* hist, int total_q,
                              int splits, int k, int32_t* out_idx, float* out_val, int* status, cudaStream_t stream,
                              const int* ok) {
  const NvtxRange nvtx("dsa.decode_merge");
  if (splits < 1 || splits > 256) return DSA_ERR_UNSUPPORTED;
  const size_t dyn = (size_t)splits * 16 * (sizeof(const uint2*) + sizeof(int));
  const size_t total = dyn + sizeof(MergeSmem) + 64;
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DSA_ERR_CUDA;
  if (total > 48 * 1024 && !(configured.load() & (uint64_t(1) << dev))) {
    if (cudaFuncSetAttribute(decode_merge_lists_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(64 * 1024 + 1024)) != cudaSuccess)
      return DSA_ERR_CUDA;
    configured.fetch_or(uint64_t(1) << dev);
  }
  decode_merge_lists_kernel<<<total_q, kMergeListThreads, dyn, stream>>>(cand, cand_cap, hdr, hist, splits, k,
                                                                         out_idx, out_val, status, ok);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Device check of a decode batch's offsets, before any kernel that reads them
// (the group form in decode runs several).  Sequence b: k_off[b] >= 0,
// 1 <= N_b = k_off[b+1] - k_off[b] <= max_keys, k_off[b+1] <= total_keys,
// q_off[b] >= 0, 1 <= m_b = q_off[b+1] - q_off[b] <= min(4, N_b), and
// q_off[B] = total_q.  Writes the verdict to hdr->offsets_ok; a failure is
// also recorded as an invalid argument in the status word.
// ---------------------------------------------------------------------------
__global__ void decode_offsets_check_kernel(const int64_t* __restrict__ k_off, const int32_t* __restrict__ q_off,
                                            int B, int64_t total_keys, int total_q, int max_keys, WsHeader* hdr) {
  bool ok = true;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int64_t k0 = k_off[b], k1 = k_off[b + 1];
    const int64_t q0 = q_off[b], q1 = q_off[b + 1];
    ok = ok && k0 >= 0 && k1 - k0 >= 1 && k1 - k0 <= max_keys && k1 <= total_keys && q0 >= 0 && q1 - q0 >= 1 &&
         q1 - q0 <= 4 && q1 - q0 <= k1 - k0;
  }
  if (threadIdx.x == 0) ok = ok && q_off[B] == total_q;
  ok = __syncthreads_and(ok) != 0;
  if (threadIdx.x == 0) {
    hdr->offsets_ok = ok ? 1 : 0;
    if (!ok) report_error(&hdr->status, DSA_ERR_INVALID_ARG, 6);
  }
}

int launch_decode_offsets_check(const int64_t* k_off, const int32_t* q_off, int B, int64_t total_keys, int total_q,
                                int max_keys, void* workspace, cudaStream_t stream) {
  const NvtxRange nvtx("dsa.decode_offsets_check");
  decode_offsets_check_kernel<<<1, 256, 0, stream>>>(k_off, q_off, B, total_keys, total_q, max_keys,
                                                     static_cast<WsHeader*>(workspace));
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
  const NvtxRange nvtx("dsa.e4m3_to_bf16");
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
  const NvtxRange nvtx("dsa.fill_scores");
  fill_neg_inf_kernel<<<592, 256, 0, stream>>>(S, n);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
