// dsa_tc.cu — tensor-core (tcgen05 / TMEM / TMA) lightning-indexer kernel.
//
// Computes I[t, s] = sum_h w[t,h] * ReLU(q[t,h,:] . k[s,:]) for bf16 q/k with
// H = 64 heads and d = 128 and keeps each query's top-k, without ever writing
// the score matrix.  The contraction q[t,h,:] . k[s,:] is a GEMM with
// M = keys, N = (query, head) columns, K = d:
//
//   * one persistent CTA per SM; a work unit is up to 4 queries (N = 4 x 64
//     = 256 columns) against the keys they see, streamed in tiles of 128;
//   * warp 8 issues TMA loads (no multicast): the unit's Q block once, then
//     key tiles into a 3-stage ring (128B-swizzled, K-major);
//   * warp 9 allocates 512 TMEM columns and issues tcgen05.mma
//     (M=128, N=nq*64, K=16 steps) into one of two 256-column accumulators;
//   * warps 0-7 (two warpgroups) drain TMEM with tcgen05.ld: each thread owns
//     one key row, so ReLU, the head weighting and the head sum stay in
//     registers; the causal cut and the streaming top-k filter follow at once.
//
// Work units come in two kinds: prefill rows (dense queries or group proxies,
// each row with its own causal position) and decode segments (the m new
// queries of one sequence against one slice of that sequence's key cache,
// whose local top-k lists a merge kernel combines).
#include "dsa_common.cuh"
#include "dsa_topk.cuh"
#include "dsa_internal.h"

namespace dsa {

constexpr int kTcThreads = 320;
constexpr int kQB = 4;            // queries per unit
constexpr int kHeads = 64;
constexpr int kTileKeys = 128;
constexpr int kStages = 3;
constexpr int kStageCap = 2048;   // staged entries of the threshold bin, per warpgroup
constexpr int kQChunkBytes = kQB * kHeads * 64 * 2;      // 32 KB: 256 rows x 128 B
constexpr int kQHeadBlockBytes = kHeads * 64 * 2;        // 8 KB: one query, one d-chunk
constexpr int kKChunkBytes = kTileKeys * 64 * 2;         // 16 KB
constexpr int kKStageBytes = 2 * kKChunkBytes;           // 32 KB

struct TcSmem {
  uint8_t q[2 * kQChunkBytes];                 // d-chunk-major: [2][256 rows][128 B]
  uint8_t k[kStages][kKStageBytes];            // [stage][2][128 rows][128 B]
  RowState rows[kQB];
  float w[kQB][kHeads];
  uint2 stage[2][kStageCap];
  uint64_t q_full, q_empty, drain;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t t_full[2], t_empty[2];
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kTcSmemBytes = sizeof(TcSmem) + 1024;  // + alignment slack

struct UnitInfo {
  int nq;            // queries in the unit (0 = no unit)
  int row0;          // first Q row
  int key_row0;      // first K row of the streamed key range (global row)
  int tile0;         // first key tile (local to the key range)
  int ntiles;        // tiles streamed
  int nkeys;         // keys in the range (local index < nkeys is valid)
  int64_t pos[kQB];  // causal position of each query (local key index)
  int seq_split;     // decode: output slot (row * splits + split); prefill: -1
};

__device__ __forceinline__ int64_t prefill_pos(const TcArgs& a, int r) {
  int64_t v = (int64_t)r * a.pos_mul + a.pos_add;
  if (v > a.pos_clamp) v = a.pos_clamp;
  return a.pos_base + v;
}

// Zig-zag, longest-first static schedule over the persistent grid.
__device__ __forceinline__ bool unit_at(const TcArgs& a, int round, UnitInfo& u) {
  const int G = gridDim.x, c = blockIdx.x;
  const int v = round * G + ((round & 1) ? (G - 1 - c) : c);
  if (v >= a.n_units) return false;
  if (a.kind == 0) {
    const int unit = a.n_units - 1 - v;
    u.row0 = unit * kQB;
    u.nq = min(kQB, a.n_rows - u.row0);
    for (int j = 0; j < kQB; ++j) u.pos[j] = prefill_pos(a, u.row0 + min(j, u.nq - 1));
    const int64_t maxpos = u.pos[u.nq - 1];
    u.key_row0 = 0;
    u.tile0 = 0;
    u.ntiles = (int)(maxpos / kTileKeys) + 1;
    u.nkeys = (int)(maxpos + 1);
    u.seq_split = -1;
  } else if (a.kind == 1) {
    const int b = v / a.splits, sp = v % a.splits;
    const int64_t k0 = a.k_off[b], k1 = a.k_off[b + 1];
    const int q0 = a.q_off[b], q1 = a.q_off[b + 1];
    const int nb = (int)(k1 - k0), mb = q1 - q0;
    u.row0 = q0;
    u.nq = mb;
    for (int j = 0; j < kQB; ++j) u.pos[j] = (int64_t)nb - mb + min(j, mb - 1);
    const int tiles_b = (nb + kTileKeys - 1) / kTileKeys;
    const int t0 = min(tiles_b, sp * a.tiles_per_split);
    const int t1 = min(tiles_b, t0 + a.tiles_per_split);
    u.key_row0 = (int)k0;
    u.tile0 = t0;
    u.ntiles = t1 - t0;
    u.nkeys = nb;
    u.seq_split = sp;
  } else {
    // group refine: members of group g against the group's gathered bank
    const int unit = a.n_units - 1 - v;
    const int g = unit / a.mblocks, mbk = unit % a.mblocks;
    const int r_end = min(a.T, (g + 1) * a.group);
    u.row0 = g * a.group + mbk * kQB;
    u.nq = max(0, min(kQB, r_end - u.row0));
    for (int j = 0; j < kQB; ++j) u.pos[j] = a.pos_base + u.row0 + min(j, max(u.nq - 1, 0));
    const int64_t L = a.pos_base + r_end - 1;
    const int nbk = (int)min((int64_t)a.bank, L + 1);
    u.key_row0 = g * a.bank;
    u.tile0 = 0;
    u.ntiles = u.nq > 0 ? (nbk + kTileKeys - 1) / kTileKeys : 0;
    u.nkeys = nbk;
    u.seq_split = g;
  }
  return true;
}

__device__ __forceinline__ bool group_and(int bar, int nthr, bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok), "r"(bar), "r"(nthr)
      : "memory");
  return r != 0;
}

__global__ void __launch_bounds__(kTcThreads, 1)
    tc_index_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  TcSmem& S = *reinterpret_cast<TcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &S.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&S.q_full, 1);
    mbar_init(&S.q_empty, 1);
    mbar_init(&S.drain, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.k_full[s], 1);
      mbar_init(&S.k_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.t_full[b], 1);
      mbar_init(&S.t_empty[b], 8);
    }
    S.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) tmem_alloc(&S.tmem_base, 512);
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;

  if (warp == 8) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int qi = 0;
      bool armed[kStages] = {};
      uint32_t armed_ph[kStages] = {};
      bool ok = true;
      UnitInfo u;
      for (int round = 0; ok && unit_at(a, round, u); ++round) {
        if (qi > 0 && !(ok = mbar_wait(&S.q_empty, (qi - 1) & 1, abort_flag, a.status, 10))) break;
        mbar_arrive_expect_tx(&S.q_full, (uint32_t)(u.nq * 2 * kQHeadBlockBytes));
        for (int q = 0; q < u.nq; ++q)
          for (int c = 0; c < 2; ++c)
            tma_load_2d(S.q + c * kQChunkBytes + q * kQHeadBlockBytes, &tmQ, &S.q_full, c * 64,
                        (u.row0 + q) * kHeads);
        ++qi;
        for (int j = 0; j < u.ntiles; ++j) {
          if (!(ok = mbar_wait(&S.k_empty[s], ph ^ 1u, abort_flag, a.status, 11))) break;
          mbar_arrive_expect_tx(&S.k_full[s], (uint32_t)kKStageBytes);
          const int row = u.key_row0 + (u.tile0 + j) * kTileKeys;
          for (int c = 0; c < 2; ++c)
            tma_load_2d(S.k[s] + c * kKChunkBytes, &tmK, &S.k_full[s], c * 64, row);
          armed[s] = true;
          armed_ph[s] = ph;
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // never leave with a copy in flight
      for (int t = 0; t < kStages; ++t)
        if (armed[t]) mbar_wait(&S.k_full[t], armed_ph[t], abort_flag, a.status, 12);
      if (qi > 0) mbar_wait(&S.q_full, (qi - 1) & 1, abort_flag, a.status, 13);
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int qi = 0, buf = 0;
      uint32_t tph[2] = {0u, 0u};
      bool ok = true;
      UnitInfo u;
      const uint32_t q_addr = smem_u32(S.q);
      for (int round = 0; ok && unit_at(a, round, u); ++round) {
        if (!(ok = mbar_wait(&S.q_full, qi & 1, abort_flag, a.status, 20))) break;
        ++qi;
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(128, u.nq * kHeads);
        for (int j = 0; j < u.ntiles; ++j) {
          if (!(ok = mbar_wait(&S.k_full[s], ph, abort_flag, a.status, 21))) break;
          if (!(ok = mbar_wait(&S.t_empty[buf], tph[buf] ^ 1u, abort_flag, a.status, 22))) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)(buf * 256);
          const uint32_t k_addr = smem_u32(S.k[s]);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sw128_kmajor_desc(k_addr + c * kKChunkBytes + kk * 32);
              const uint64_t bd = sw128_kmajor_desc(q_addr + c * kQChunkBytes + kk * 32);
              tc_mma_bf16(d_tmem, ad, bd, idesc, (c | kk) != 0);
            }
          }
          tc_commit(&S.k_empty[s]);
          tc_commit(&S.t_full[buf]);
          tph[buf] ^= 1u;
          buf ^= 1;
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&S.q_empty);
      }
      // never leave with an MMA in flight
      tc_commit(&S.drain);
      mbar_wait(&S.drain, 0, abort_flag, a.status, 23);
    }
  } else {
    // ---------------- epilogue: warps 0-7, two warpgroups ----------------
    const int wg = warp >> 2, lq = warp & 3, tid = threadIdx.x & 127;
    const int bar = 1 + wg;
    uint32_t eph[2] = {0u, 0u};
    int buf = 0;
    UnitInfo u;
    bool ok = true;
    for (int round = 0; ok && unit_at(a, round, u); ++round) {
      // my query slots: wg, wg + 2
      const int ns = (u.nq > wg) + (u.nq > wg + 2);
      for (int j = 0; j < ns; ++j) {
        const int slot = wg + 2 * j;
        row_reset(S.rows[slot], tid, 128);
        if (tid < kHeads) S.w[slot][tid] = a.w[(int64_t)(u.row0 + slot) * kHeads + tid];
      }
      // causal positions of my two slots (constant indices keep them in registers)
      int64_t mypos[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) mypos[j] = (wg == 0) ? u.pos[2 * j] : u.pos[2 * j + 1];
      named_bar(bar, 128);
      int64_t cslot_base = (int64_t)blockIdx.x * kQB;
      for (int jt = 0; jt < u.ntiles; ++jt) {
        bool w_ok = mbar_wait(&S.t_full[buf], eph[buf], abort_flag, a.status, 30);
        if (!group_and(bar, 128, w_ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float v[2][64];
        const uint32_t lane_base = (uint32_t)(lq * 32) << 16;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (j < ns) {
            const uint32_t col = (uint32_t)(buf * 256 + (wg + 2 * j) * kHeads);
            tmem_ld_32x32b_x32(tmem_base + lane_base + col, &v[j][0]);
            tmem_ld_32x32b_x32(tmem_base + lane_base + col + 32, &v[j][32]);
          }
        }
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.t_empty[buf]);
        eph[buf] ^= 1u;
        buf ^= 1;

        const int key = (u.tile0 + jt) * kTileKeys + lq * 32 + lane;  // local key index
        const bool in_range = key < u.nkeys;
        int64_t kpos = key;
        if (a.kind == 2) kpos = in_range ? (int64_t)a.key_map[(int64_t)u.seq_split * a.bank + key] : -1;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (j < ns) {
            const int slot = wg + 2 * j;
            const float4* w4 = reinterpret_cast<const float4*>(S.w[slot]);
            float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
            for (int h = 0; h < kHeads; h += 4) {
              const float4 ww = w4[h >> 2];
              s0 = fmaf(ww.x, fmaxf(v[j][h + 0], 0.f), s0);
              s1 = fmaf(ww.y, fmaxf(v[j][h + 1], 0.f), s1);
              s2 = fmaf(ww.z, fmaxf(v[j][h + 2], 0.f), s2);
              s3 = fmaf(ww.w, fmaxf(v[j][h + 3], 0.f), s3);
            }
            float score = (s0 + s1) + (s2 + s3);
            score = score + 0.0f;  // -0 -> +0
            const bool valid = in_range && kpos >= 0 && kpos <= mypos[j];
            if (a.dbg_scores != nullptr && valid)
              a.dbg_scores[(int64_t)(u.row0 + slot) * a.dbg_ld + kpos] = score;
            uint2* cand = a.cand + (cslot_base + slot) * a.cand_cap;
            row_append(S.rows[slot], cand, score, (uint32_t)kpos, valid, lane);
          }
        }
        named_bar(bar, 128);
        if (lq < ns) row_update(S.rows[wg + 2 * lq], a.k, lane);
        named_bar(bar, 128);
      }
      if (!ok) break;
      // final selection for my slots
      for (int j = 0; j < ns; ++j) {
        const int slot = wg + 2 * j;
        const uint2* cand = a.cand + (cslot_base + slot) * a.cand_cap;
        int32_t* oi;
        float* ov;
        if (a.kind != 1) {
          oi = a.out_idx + (int64_t)(u.row0 + slot) * a.out_ld;
          ov = a.out_val + (int64_t)(u.row0 + slot) * a.out_ld;
        } else {
          const int64_t o = ((int64_t)(u.row0 + slot) * a.splits + u.seq_split);
          oi = a.out_idx + o * a.out_ld;
          ov = a.out_val + o * a.out_ld;
        }
        const int cnt = row_select(S.rows[slot], cand, a.k, oi, ov, S.stage[wg], kStageCap, tid, 128, bar,
                                   a.status);
        if (a.kind == 1 && tid == 0) a.out_cnt[(int64_t)(u.row0 + slot) * a.splits + u.seq_split] = cnt;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem_base, 512);
}

int launch_tc_index(const CUtensorMap& tmQ, const CUtensorMap& tmK, const TcArgs& a, int grid,
                    cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(tc_index_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kTcSmemBytes) != cudaSuccess)
      return DSA_ERR_CUDA;
    configured = true;
  }
  tc_index_kernel<<<grid, kTcThreads, kTcSmemBytes, stream>>>(tmQ, tmK, a);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

size_t tc_smem_bytes() { return kTcSmemBytes; }

}  // namespace dsa
