// dsa_ivf.cu — plain k-means index build for inverted-file routing.
//
// The keys are grouped by similarity with Lloyd iterations (centroid i
// starts at key floor(i N / C); every key goes to its nearest centroid, ties
// to the lower one; every centroid moves to its members' mean, an empty one
// stays), then laid out cluster after cluster so that a routed query reads
// each probed cluster as contiguous TMA tiles.  Index layout (one buffer):
//   off [C+1] int32, perm [N] int32 (sorted row -> key), assign [N] int32,
//   keys [N, d] bf16 (sorted; fp8 keys widened, their scale stays per key),
//   centroids [C, d] bf16 (routing) and fp32.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

namespace {

__device__ __forceinline__ float key_elem(const __nv_bfloat16* K, const float* ks, int64_t r, int d, int j) {
  const float x = __bfloat162float(K[r * d + j]);
  return ks ? x * ks[r] : x;
}

__global__ void ivf_init_kernel(const __nv_bfloat16* __restrict__ K, const float* __restrict__ ks, int64_t N, int d,
                                int C, float* __restrict__ cen) {
  const int c = blockIdx.x;
  const int64_t r = ((int64_t)c * N) / C;
  for (int j = threadIdx.x; j < d; j += blockDim.x) cen[(int64_t)c * d + j] = key_elem(K, ks, r, d, j);
}

__global__ void ivf_norm_kernel(const float* __restrict__ cen, int C, int d, float* __restrict__ norm) {
  const int c = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (c >= C) return;
  float s = 0.f;
  for (int j = lane; j < d; j += 32) s = fmaf(cen[(int64_t)c * d + j], cen[(int64_t)c * d + j], s);
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) norm[c] = s;
}

// One warp per key: lane l holds elements l, l+32, .. (d <= 256); the
// nearest centroid minimises |c|^2 - 2 k.c (|k|^2 is common to all), first
// minimum kept.
__global__ void ivf_assign_kernel(const __nv_bfloat16* __restrict__ K, const float* __restrict__ ks, int64_t N,
                                  int d, const float* __restrict__ cen, const float* __restrict__ norm, int C,
                                  int32_t* __restrict__ assign) {
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= N) return;
  float x[8];
  const int m = d / 32;
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = e < m ? key_elem(K, ks, r, d, lane + 32 * e) : 0.f;
  float best = 0.f;
  int bi = 0;
  for (int c = 0; c < C; ++c) {
    const float* cc = cen + (int64_t)c * d;
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (e < m) s = fmaf(x[e], cc[lane + 32 * e], s);
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float dist = norm[c] - 2.f * s;
    if (c == 0 || dist < best) {
      best = dist;
      bi = c;
    }
  }
  if (lane == 0) assign[r] = bi;
}

// The same assignment as a tiled product: a block takes 64 keys against the
// centroids 64 at a time, d in chunks of 32 staged in shared memory, each
// thread 4 keys x 4 centroids; the nearest centroid (lowest index among
// equals) is kept per key across tiles and then across the 16 threads that
// share a key.  d must be a multiple of 32.
constexpr int kAsgKeys = 64, kAsgCen = 64, kAsgD = 32;

__global__ void __launch_bounds__(256) ivf_assign_tiled_kernel(const __nv_bfloat16* __restrict__ K,
                                                               const float* __restrict__ ks, int64_t N, int d,
                                                               const float* __restrict__ cen,
                                                               const float* __restrict__ norm, int C,
                                                               int32_t* __restrict__ assign) {
  // chunks stored transposed; rows padded by 4 floats (16-byte reads stay
  // aligned, the transposing stores spread over 8 banks instead of one)
  __shared__ __align__(16) float As[kAsgD][kAsgKeys + 4];
  __shared__ __align__(16) float Bs[kAsgD][kAsgCen + 4];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t r0 = (int64_t)blockIdx.x * kAsgKeys;
  float best[4];
  int bi[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    best[i] = __int_as_float(0x7f800000);
    bi[i] = 0x7fffffff;
  }
  for (int c0 = 0; c0 < C; c0 += kAsgCen) {
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int l = 0; l < 4; ++l) acc[i][l] = 0.f;
    for (int j0 = 0; j0 < d; j0 += kAsgD) {
      for (int e = tid; e < kAsgKeys * kAsgD; e += 256) {
        const int r = e / kAsgD, j = e % kAsgD;
        const int64_t row = r0 + r;
        As[j][r] = row < N ? key_elem(K, ks, row, d, j0 + j) : 0.f;
      }
      for (int e = tid; e < kAsgCen * kAsgD; e += 256) {
        const int c = e / kAsgD, j = e % kAsgD;
        Bs[j][c] = c0 + c < C ? cen[(int64_t)(c0 + c) * d + j0 + j] : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int j = 0; j < kAsgD; ++j) {
        const float4 a = *reinterpret_cast<const float4*>(&As[j][ty * 4]);
        const float4 b = *reinterpret_cast<const float4*>(&Bs[j][tx * 4]);
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int l = 0; l < 4; ++l) acc[i][l] = fmaf(av[i], bv[l], acc[i][l]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int l = 0; l < 4; ++l) {
      const int c = c0 + tx * 4 + l;
      if (c < C) {
        const float nc = norm[c];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float dist = nc - 2.f * acc[i][l];
          if (dist < best[i]) {  // centroids arrive in increasing order: the first minimum stays
            best[i] = dist;
            bi[i] = c;
          }
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best[i], o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi[i], o);
      if (ob < best[i] || (ob == best[i] && oi < bi[i])) {
        best[i] = ob;
        bi[i] = oi;
      }
    }
    const int64_t row = r0 + ty * 4 + i;
    if (tx == 0 && row < N) assign[row] = bi[i];
  }
}

__global__ void ivf_accumulate_kernel(const __nv_bfloat16* __restrict__ K, const float* __restrict__ ks, int64_t N,
                                      int d, const int32_t* __restrict__ assign, float* __restrict__ sum,
                                      int32_t* __restrict__ count) {
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= N) return;
  const int c = assign[r];
  for (int j = lane; j < d; j += 32) atomicAdd(&sum[(int64_t)c * d + j], key_elem(K, ks, r, d, j));
  if (lane == 0) atomicAdd(&count[c], 1);
}

__global__ void ivf_update_kernel(const float* __restrict__ sum, const int32_t* __restrict__ count, int C, int d,
                                  float* __restrict__ cen, __nv_bfloat16* __restrict__ cen_bf16) {
  const int c = blockIdx.x;
  const int n = count[c];
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    if (n > 0) cen[(int64_t)c * d + j] = sum[(int64_t)c * d + j] / (float)n;
    if (cen_bf16) cen_bf16[(int64_t)c * d + j] = __float2bfloat16_rn(cen[(int64_t)c * d + j]);
  }
}

// Exclusive scan of the cluster sizes (one block).
__global__ void ivf_offsets_kernel(const int32_t* __restrict__ count, int C, int32_t* __restrict__ off) {
  __shared__ int part[1024];
  const int tid = threadIdx.x, per = (C + 1023) / 1024;
  const int c0 = tid * per, c1 = min(C, c0 + per);
  int s = 0;
  for (int c = c0; c < c1; ++c) s += count[c];
  part[tid] = s;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    const int v = tid >= o ? part[tid - o] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int acc = part[tid] - s;
  for (int c = c0; c < c1; ++c) {
    off[c] = acc;
    acc += count[c];
  }
  if (tid == 1023) off[C] = part[1023];
}

// Key r goes to row off[c] + (a slot taken in arrival order) of its cluster.
__global__ void ivf_scatter_kernel(const uint4* __restrict__ K, int row_vecs, int64_t N,
                                   const int32_t* __restrict__ assign, const int32_t* __restrict__ off,
                                   int32_t* __restrict__ cursor, int32_t* __restrict__ perm,
                                   uint4* __restrict__ Ks) {
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= N) return;
  int dst = 0;
  if (lane == 0) {
    const int c = assign[r];
    dst = off[c] + atomicAdd(&cursor[c], 1);
    perm[dst] = (int32_t)r;
  }
  dst = __shfl_sync(0xffffffffu, dst, 0);
  for (int v = lane; v < row_vecs; v += 32) Ks[(int64_t)dst * row_vecs + v] = K[r * row_vecs + v];
}

// Tiles a routed query streams: sum over its probed clusters of ceil(size / 128).
__global__ void ivf_tiles_kernel(const int32_t* __restrict__ list, int n_probe, int T,
                                 const int32_t* __restrict__ off, int32_t* __restrict__ tiles) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  int n = 0;
  for (int i = 0; i < n_probe; ++i) {
    const int c = list[(int64_t)t * n_probe + i];
    if (c >= 0) n += (off[c + 1] - off[c] + 127) / 128;
  }
  tiles[t] = n;
}

}  // namespace

IvfIndex ivf_index_view(void* base, int64_t N, int d, int C) {
  IvfIndex x;
  uint8_t* p = static_cast<uint8_t*>(base);
  auto take = [&](size_t bytes) {
    uint8_t* q = p;
    p += (bytes + 255) & ~size_t(255);
    return q;
  };
  x.off = reinterpret_cast<int32_t*>(take((size_t)(C + 1) * 4));
  x.perm = reinterpret_cast<int32_t*>(take((size_t)N * 4));
  x.assign = reinterpret_cast<int32_t*>(take((size_t)N * 4));
  x.keys = take((size_t)N * d * 2);
  x.cen_bf16 = take((size_t)C * d * 2);
  x.cen = reinterpret_cast<float*>(take((size_t)C * d * 4));
  x.bytes = (size_t)(p - static_cast<uint8_t*>(base));
  return x;
}

size_t ivf_build_scratch_bytes(int d, int C) { return (size_t)C * d * 4 + (size_t)C * 4 * 3 + 1024; }

int ivf_build(const void* K, const float* K_scale, int64_t N, int d, int C, int iters, const IvfIndex& x,
              uint8_t* scratch, cudaStream_t st) {
  const NvtxRange nvtx("dsa.ivf_build");
  const __nv_bfloat16* Kb = static_cast<const __nv_bfloat16*>(K);
  float* sum = reinterpret_cast<float*>(scratch);
  int32_t* count = reinterpret_cast<int32_t*>(sum + (size_t)C * d);
  int32_t* cursor = count + C;
  float* norm = reinterpret_cast<float*>(cursor + C);
  const unsigned key_blocks = (unsigned)((N + 7) / 8);  // 8 warps per block, a warp per key
  ivf_init_kernel<<<C, 128, 0, st>>>(Kb, K_scale, N, d, C, x.cen);
  for (int it = 0; it < iters; ++it) {
    ivf_norm_kernel<<<(C + 7) / 8, 256, 0, st>>>(x.cen, C, d, norm);
    if (d % kAsgD == 0)
      ivf_assign_tiled_kernel<<<(unsigned)((N + kAsgKeys - 1) / kAsgKeys), 256, 0, st>>>(Kb, K_scale, N, d, x.cen,
                                                                                          norm, C, x.assign);
    else
      ivf_assign_kernel<<<key_blocks, 256, 0, st>>>(Kb, K_scale, N, d, x.cen, norm, C, x.assign);
    if (cudaMemsetAsync(sum, 0, (size_t)C * d * 4 + (size_t)C * 4, st) != cudaSuccess) return DSA_ERR_CUDA;
    ivf_accumulate_kernel<<<key_blocks, 256, 0, st>>>(Kb, K_scale, N, d, x.assign, sum, count);
    ivf_update_kernel<<<C, 128, 0, st>>>(sum, count, C, d, x.cen, it + 1 == iters ? (__nv_bfloat16*)x.cen_bf16 : nullptr);
  }
  ivf_offsets_kernel<<<1, 1024, 0, st>>>(count, C, x.off);
  if (cudaMemsetAsync(cursor, 0, (size_t)C * 4, st) != cudaSuccess) return DSA_ERR_CUDA;
  ivf_scatter_kernel<<<key_blocks, 256, 0, st>>>(static_cast<const uint4*>(K), d * 2 / 16, N, x.assign, x.off,
                                                  cursor, x.perm, static_cast<uint4*>(x.keys));
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

int launch_ivf_tiles(const int32_t* list, int n_probe, int T, const int32_t* off, int32_t* tiles, cudaStream_t st) {
  const NvtxRange nvtx("dsa.ivf_tiles");
  ivf_tiles_kernel<<<(T + 255) / 256, 256, 0, st>>>(list, n_probe, T, off, tiles);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
