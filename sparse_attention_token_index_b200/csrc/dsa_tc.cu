// dsa_tc.cu — tensor-core (tcgen05 / TMEM / TMA) lightning-indexer kernel.
//
// Computes I[t, s] = sum_h w[t,h] * ReLU(q[t,h,:] . k[s,:]) for bf16 q/k with
// H = 64 heads and d = 128 and keeps each query's top-k, without ever writing
// the score matrix.  The contraction q[t,h,:] . k[s,:] is a GEMM with
// M = keys, N = (query, head) columns, K = d:
//
//   * one persistent CTA per SM; a work unit is up to 4 queries (N = 4 x 64
//     = 256 columns) against the keys they see, streamed in tiles of 128;
//   * warp 16 issues TMA loads (no multicast): the unit's Q block once, then
//     key tiles into a 3-stage ring (128B-swizzled, K-major);
//   * warp 17 allocates 512 TMEM columns and issues tcgen05.mma
//     (M=128, N=nq*64, K=16 steps) into one of two 256-column accumulators;
//   * warps 0-15 form four epilogue warpgroups, one per query of the unit.
//     Each thread owns one key row of the tile: tcgen05.ld brings its 64 head
//     dot products into registers, ReLU and the head weights are applied with
//     packed fp32x2 FMAs, and the causal cut and the streaming top-k filter
//     follow at once.
//
// Work units come in five kinds (a template parameter): prefill rows (dense
// queries, group proxies or block-routing rows, each row with its own causal
// position), decode segments (the m new queries of one sequence against one
// slice of that sequence's key cache; a merge kernel combines the slices),
// group-refine blocks (up to 4 members of a group against the group's
// gathered candidate bank), and the refine stages of the two routing
// comparators (one query against its routed key blocks, or against its
// probed clusters in the clustered keys).  A second template parameter marks
// scaled keys (fp8 keys widened to bf16, a per-key scale after the head sum).
#include <atomic>
#include <type_traits>

#include "dsa_common.cuh"
#include "dsa_topk.cuh"
#include "dsa_internal.h"

namespace dsa {

constexpr int kEpiWarps = 16;
constexpr int kTcThreads = (kEpiWarps + 3) * 32;  // + TMA producer + MMA issuer + threshold warp
constexpr int kProducerWarp = kEpiWarps;
constexpr int kMmaWarp = kEpiWarps + 1;
constexpr int kThreshWarp = kEpiWarps + 2;
constexpr int kQB = 4;            // queries per unit
constexpr int kHeads = 64;
constexpr int kTileKeys = 128;
constexpr int kStages = 3;
constexpr int kStageCap = 1024;   // staged entries of the threshold bin, per query
constexpr int kQChunkBytes = kQB * kHeads * 64 * 2;      // 32 KB: 256 rows x 128 B
constexpr int kQHeadBlockBytes = kHeads * 64 * 2;        // 8 KB: one query, one d-chunk
constexpr int kKChunkBytes = kTileKeys * 64 * 2;         // 16 KB
constexpr int kKStageBytes = 2 * kKChunkBytes;           // 32 KB

struct TcSmem {
  uint8_t q[2 * kQChunkBytes];                 // d-chunk-major: [2][256 rows][128 B]
  uint8_t k[kStages][kKStageBytes];            // [stage][2][128 rows][128 B]
  RowState rows[kQB];
  float w[kQB][kHeads];
  uint2 stage[kQB][kStageCap];
  uint64_t q_full, q_empty, drain;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t t_full[2], t_empty[2];
  uint32_t tmem_base;
  int abort_flag;
  int epi_done;  // epilogue warpgroups that left their unit loop
};

constexpr size_t kTcSmemBytes = sizeof(TcSmem) + 1024;  // + alignment slack
static_assert(kTcSmemBytes <= 232448, "fits the 227 KB opt-in shared memory of one CTA");

struct UnitInfo {
  int nq;            // queries in the unit (0 = no work)
  int row0;          // first Q row
  int key_row0;      // first K row of the streamed key range (global row)
  int tile0;         // first key tile (local to the key range)
  int ntiles;        // tiles streamed
  int nkeys;         // keys in the range (local index < nkeys is valid)
  int seq_split;     // decode: split; refine: group index
  int partial;       // decode: leaves a partial list
  int pos0;          // refine / routed: causal position of the unit's first query
  int rsel;          // routed: routed blocks streamed first
  int rown;          // routed: the query's own partial block, streamed last
};

// Sorted-key rows an inverted-file unit streams: its probed clusters one after
// the other, 128 rows a tile (a cluster's last tile is cut at the cluster's
// end).  The producer and the epilogue each step one through every tile.
struct ClusterWalk {
  const int32_t* list;
  int n, ci, row, end;
  __device__ __forceinline__ void seek(const TcArgs& a) {  // first non-empty cluster from ci on
    while (ci < n) {
      const int c = list[ci];
      row = c >= 0 ? a.ivf_off[c] : 0;
      end = c >= 0 ? a.ivf_off[c + 1] : 0;
      if (row < end) return;
      ++ci;
    }
    row = end = 0;
  }
  __device__ __forceinline__ void start(const TcArgs& a, int t) {
    list = a.route_blocks + (int64_t)t * a.route_n;
    n = a.route_n;
    ci = 0;
    seek(a);
  }
  __device__ __forceinline__ void next(const TcArgs& a) {
    row += 128;
    if (row >= end) {
      ++ci;
      seek(a);
    }
  }
};

// Key block of iteration j of a routed unit: its routed blocks, then its own.
__device__ __forceinline__ int routed_block(const TcArgs& a, const UnitInfo& u, int j) {
  return j < u.rsel ? a.route_blocks[(int64_t)u.row0 * a.route_n + j] : u.rown;
}

__device__ __forceinline__ int64_t prefill_pos(const TcArgs& a, int r) {
  if (a.pos_shift > 0) return ((a.pos_base + r + 1) >> a.pos_shift) - 1;
  int64_t v = (int64_t)r * a.pos_mul + a.pos_add;
  if (v > a.pos_clamp) v = a.pos_clamp;
  return a.pos_base + v;
}

// Zig-zag, longest-first static schedule over the persistent grid.
template <int kKind>
__device__ __forceinline__ bool unit_at(const TcArgs& a, int round, UnitInfo& u) {
  const int G = gridDim.x, c = blockIdx.x;
  const int v = round * G + ((round & 1) ? (G - 1 - c) : c);
  if (v >= a.n_units) return false;
  if constexpr (kKind == 0) {
    const int unit = a.n_units - 1 - v;
    u.row0 = unit * kQB;
    u.nq = min(kQB, a.n_rows - u.row0);
    const int64_t maxpos = prefill_pos(a, u.row0 + u.nq - 1);
    u.key_row0 = 0;
    u.tile0 = 0;
    u.ntiles = maxpos >= 0 ? (int)(maxpos / kTileKeys) + 1 : 0;
    u.nkeys = (int)(maxpos + 1);
    u.seq_split = -1;
    u.partial = 0;
  } else if constexpr (kKind == 4) {
    // inverted-file refine: one query row over its probed clusters (longest first)
    const int t = a.n_units - 1 - v;
    u.row0 = t;
    u.nq = 1;
    u.key_row0 = 0;
    u.tile0 = 0;
    u.ntiles = a.ivf_tiles[t];
    if (u.ntiles > a.ivf_max_tiles) {  // more tiles than the candidate lists hold: report, stay in bounds
      if (threadIdx.x == 0) report_error(a.status, DSA_ERR_INTERNAL, 5);
      u.ntiles = a.ivf_max_tiles;
    }
    u.nkeys = 0;  // rows are checked against their cluster's end
    u.seq_split = -1;
    u.partial = 0;
    u.pos0 = (int)(a.pos_base + t);
  } else if constexpr (kKind == 3) {
    // routed refine: one query row over its routed blocks (longest first)
    const int t = a.n_units - 1 - v;
    const int64_t p = a.pos_base + t;
    const int own = (int)((p + 1) / kTileKeys);  // complete blocks before the query
    u.row0 = t;
    u.nq = 1;
    u.rsel = min(a.route_n, own);
    u.rown = own;
    u.key_row0 = 0;
    u.tile0 = 0;
    u.ntiles = u.rsel + (((int64_t)own * kTileKeys <= p) ? 1 : 0);  // own block non-empty
    u.nkeys = (int)(p + 1);
    u.seq_split = -1;
    u.partial = 0;
    u.pos0 = (int)p;
  } else if constexpr (kKind == 1) {
    const int b = v / a.splits, sp = v % a.splits;
    const int64_t k0 = a.k_off[b], k1 = a.k_off[b + 1];
    // no query offsets: one query row per sequence (decode proxies)
    const int q0 = a.q_off ? a.q_off[b] : b, q1 = a.q_off ? a.q_off[b + 1] : b + 1;
    // the sequence must lie inside K and Q, fit this plan's slices
    // (N_b <= max_keys) and have 1 <= m_b <= min(4, N_b); otherwise the unit
    // does nothing and the call reports an invalid argument
    const int64_t nb64 = k1 - k0;
    const bool seq_ok = k0 >= 0 && nb64 >= 1 && k1 <= a.total_keys &&
                        nb64 <= (int64_t)a.splits * a.tiles_per_split * kTileKeys && q0 >= 0 && q1 <= a.n_rows &&
                        q1 - q0 >= 1 && q1 - q0 <= kQB && (int64_t)(q1 - q0) <= nb64;
    const int nb = seq_ok ? (int)nb64 : 0;
    u.row0 = seq_ok ? q0 : 0;
    u.nq = seq_ok ? q1 - q0 : 0;
    const int tiles_b = (nb + kTileKeys - 1) / kTileKeys;
    const int t0 = min(tiles_b, sp * a.tiles_per_split);
    const int t1 = min(tiles_b, t0 + a.tiles_per_split);
    u.key_row0 = seq_ok ? (int)k0 : 0;
    u.tile0 = t0;
    u.ntiles = t1 - t0;
    u.nkeys = nb;
    u.seq_split = sp;
    u.partial = 1;
    if (!seq_ok && threadIdx.x == 0) report_error(a.status, DSA_ERR_INVALID_ARG, 3);
  } else {
    // group refine: members of group g against the group's gathered bank
    const int unit = a.n_units - 1 - v;
    const int g = unit / a.mblocks, mbk = unit % a.mblocks;
    int nbk;
    if (a.k_off != nullptr) {
      // decode groups: group g is sequence g, its queries at N_g - m_g + j,
      // its bank indices local to the sequence
      const int q0 = a.q_off[g], q1 = a.q_off[g + 1];
      const int64_t k0 = a.k_off[g], k1 = a.k_off[g + 1];
      const bool seq_ok = k0 >= 0 && k1 - k0 >= 1 && k1 <= a.total_keys && q0 >= 0 && q1 <= a.T &&
                          q1 - q0 >= 1 && q1 - q0 <= kQB * a.mblocks && (int64_t)(q1 - q0) <= k1 - k0;
      const int nb = seq_ok ? (int)(k1 - k0) : 0;
      u.row0 = seq_ok ? q0 + mbk * kQB : 0;
      u.nq = seq_ok ? max(0, min(kQB, q1 - u.row0)) : 0;
      u.pos0 = seq_ok ? nb - (q1 - q0) + (u.row0 - q0) : 0;
      nbk = min(a.bank, nb);
      // 1 <= m_b <= min(4, N_b), sequence inside K and Q: else no work, invalid argument
      if (!seq_ok && threadIdx.x == 0) report_error(a.status, DSA_ERR_INVALID_ARG, 4);
    } else {
      const int r_end = min(a.T, (g + 1) * a.group);
      u.row0 = g * a.group + mbk * kQB;
      u.nq = max(0, min(kQB, r_end - u.row0));
      u.pos0 = (int)(a.pos_base + u.row0);
      const int64_t L = a.pos_base + r_end - 1;
      nbk = (int)min((int64_t)a.bank, L + 1);
    }
    if (a.key_slots) nbk = a.key_slots;  // query-specific additions follow the bank
    u.key_row0 = g * a.bank;
    u.tile0 = 0;
    u.ntiles = u.nq > 0 ? (nbk + kTileKeys - 1) / kTileKeys : 0;
    u.nkeys = nbk;
    u.seq_split = g;
    u.partial = 0;
  }
  return true;
}

// Causal position of query `slot` of a unit (slot < u.nq), in key-index units.
template <int kKind>
__device__ __forceinline__ int64_t slot_pos(const TcArgs& a, const UnitInfo& u, int slot) {
  if constexpr (kKind == 0) return prefill_pos(a, u.row0 + slot);
  if constexpr (kKind == 1) return (int64_t)u.nkeys - u.nq + slot;
  return (int64_t)u.pos0 + slot;  // kinds 2 and 3
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

// Two fp32 values in one 64-bit register pair, and c + a * b on both lanes
// at once (fma.rn.f32x2: per-lane IEEE fma).  Accumulators and weights stay
// in 64-bit form so that only the ReLU results need pairing.
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ float2 unpack2(uint64_t r) {
  float2 d;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(r));
  return d;
}

__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// 2 * ReLU(x) as x + |x|: one add whose |x| is an operand modifier, so it
// issues to the FMA pipe rather than the half-rate ALU pipe that a max would
// use.  Exact: 2x for x > 0 (doubling is exact), +0 otherwise.
__device__ __forceinline__ float relu_x2(float x) { return x + fabsf(x); }

// acc += (w[h] / 2) * 2 ReLU(v[h]) over 16 heads (w2 points at those heads'
// halved weights, four per 16-byte load) into one packed accumulator: even
// heads in one lane, odd heads in the other.  Scaling by 1/2 and 2 is exact,
// so each fma sees the product w[h] * ReLU(v[h]).  One serial chain is
// enough for unscaled keys: the ReLU adds and the other warps fill its
// latency, and the registers it leaves free beat parallel chains.
__device__ __forceinline__ void head_accumulate16(const float (&v)[16], const ulonglong2* __restrict__ w2,
                                                  uint64_t& acc) {
#pragma unroll
  for (int h = 0; h < 16; h += 8) {
    const ulonglong2 wa = w2[h >> 2], wb = w2[(h >> 2) + 1];
    acc = ffma2(wa.x, pack2(relu_x2(v[h + 0]), relu_x2(v[h + 1])), acc);
    acc = ffma2(wa.y, pack2(relu_x2(v[h + 2]), relu_x2(v[h + 3])), acc);
    acc = ffma2(wb.x, pack2(relu_x2(v[h + 4]), relu_x2(v[h + 5])), acc);
    acc = ffma2(wb.y, pack2(relu_x2(v[h + 6]), relu_x2(v[h + 7])), acc);
  }
}

// The sum over 32 heads in four packed accumulators (four independent
// chains).  The scaled-key kernels (fp8 keys, a per-key scale load after the
// sum) measured faster this way.
__device__ __forceinline__ void head_accumulate32(const float (&v)[32], const ulonglong2* __restrict__ w2,
                                                  uint64_t (&acc)[4]) {
#pragma unroll
  for (int h = 0; h < 32; h += 8) {
    const ulonglong2 wa = w2[h >> 2], wb = w2[(h >> 2) + 1];
    acc[0] = ffma2(wa.x, pack2(relu_x2(v[h + 0]), relu_x2(v[h + 1])), acc[0]);
    acc[1] = ffma2(wa.y, pack2(relu_x2(v[h + 2]), relu_x2(v[h + 3])), acc[1]);
    acc[2] = ffma2(wb.x, pack2(relu_x2(v[h + 4]), relu_x2(v[h + 5])), acc[2]);
    acc[3] = ffma2(wb.y, pack2(relu_x2(v[h + 6]), relu_x2(v[h + 7])), acc[3]);
  }
}

// Score pairs of the accumulators, summed.
__device__ __forceinline__ float acc_sum(uint64_t acc) {
  const float2 a0 = unpack2(acc);
  return a0.x + a0.y;
}
__device__ __forceinline__ float acc_sum(const uint64_t (&acc)[4]) {
  const float2 a0 = unpack2(acc[0]), a1 = unpack2(acc[1]), a2 = unpack2(acc[2]), a3 = unpack2(acc[3]);
  return ((a0.x + a0.y) + (a1.x + a1.y)) + ((a2.x + a2.y) + (a3.x + a3.y));
}

// kScaled: the keys carry a per-key scale (fp8 keys); the scale pointer is
// then non-null and applied after the head sum.
template <bool kDebug, int kKind, bool kScaled>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_index_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ TcArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  // 1024-byte aligned (128B-swizzled TMA tiles) by a byte offset from the
  // __shared__ array itself, so every access through S stays a shared-memory
  // access (a detour through an integer address would make them generic)
  TcSmem& S = *reinterpret_cast<TcSmem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (offsets_bad(a.offsets_ok)) return;  // the whole CTA, before any barrier or TMEM
  const uint64_t budget = a.wait_ns ? a.wait_ns : kWaitNs;  // budget of the inter-role waits
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
      mbar_init(&S.t_empty[b], kEpiWarps);
    }
    S.abort_flag = 0;
    S.epi_done = 0;
    for (int q = 0; q < kQB; ++q) S.rows[q].tb = 0u;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) tmem_alloc(&S.tmem_base, 512);
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;

  if (warp == kProducerWarp) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const uint64_t pol_first = l2_evict_first(), pol_last = l2_evict_last();
      int s = 0;
      uint32_t ph = 0;
      int qi = 0;
      uint32_t armed = 0u, armed_ph = 0u;  // bit s: stage s armed / its phase
      bool ok = true;
      UnitInfo u;
      for (int round = 0; ok && unit_at<kKind>(a, round, u); ++round) {
        if (qi > 0 && !(ok = mbar_wait<true>(&S.q_empty, (qi - 1) & 1, abort_flag, a.status, 10, budget))) break;
        mbar_arrive_expect_tx(&S.q_full, (uint32_t)(u.nq * 2 * kQHeadBlockBytes));
        for (int q = 0; q < u.nq; ++q)
          for (int c = 0; c < 2; ++c)
            tma_load_2d_hint(S.q + c * kQChunkBytes + q * kQHeadBlockBytes, &tmQ, &S.q_full, c * 64,
                             (u.row0 + q) * kHeads, pol_first);
        ++qi;
        {
          // the next unit's queries into L2 now, so that its load (issued
          // only once this unit's last MMA is done) does not wait on HBM
          UnitInfo un;
          if (unit_at<kKind>(a, round + 1, un))
            for (int q = 0; q < un.nq; ++q)
              for (int c = 0; c < 2; ++c) tma_prefetch_l2_2d(&tmQ, c * 64, (un.row0 + q) * kHeads);
        }
        ClusterWalk walk;
        if constexpr (kKind == 4) walk.start(a, u.row0);
        for (int j = 0; j < u.ntiles; ++j) {
          if (!(ok = mbar_wait<true>(&S.k_empty[s], ph ^ 1u, abort_flag, a.status, 11, budget))) break;
          if (kKind == 0 && a.hold_first_tile && blockIdx.x == 0 && round == 0 && j == 0) {
            // failure-path test: this stage is never armed nor loaded, so the
            // MMA issuer's wait for it runs out
            if (++s == kStages) {
              s = 0;
              ph ^= 1u;
            }
            continue;
          }
          mbar_arrive_expect_tx(&S.k_full[s], (uint32_t)kKStageBytes);
          int row;
          if constexpr (kKind == 4) {
            row = walk.row;
            walk.next(a);
          } else {
            row = (kKind == 3) ? routed_block(a, u, j) * kTileKeys : u.key_row0 + (u.tile0 + j) * kTileKeys;
          }
          for (int c = 0; c < 2; ++c) {
            // prefill keys are read by every unit: they stay in L2; a decode
            // cache streams by once; a gathered bank is left to the default
            if (kKind == 1)
              tma_load_2d_hint(S.k[s] + c * kKChunkBytes, &tmK, &S.k_full[s], c * 64, row, pol_first);
            else if (kKind == 2)
              tma_load_2d(S.k[s] + c * kKChunkBytes, &tmK, &S.k_full[s], c * 64, row);
            else
              tma_load_2d_hint(S.k[s] + c * kKChunkBytes, &tmK, &S.k_full[s], c * 64, row, pol_last);
          }
          armed |= 1u << s;
          armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // never leave with a copy in flight
      for (int t = 0; t < kStages; ++t)
        if ((armed >> t) & 1u) mbar_wait_drain(&S.k_full[t], (armed_ph >> t) & 1u, a.status, 12);
      if (qi > 0) mbar_wait_drain(&S.q_full, (qi - 1) & 1, a.status, 13);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int qi = 0, buf = 0;
      uint32_t tph = 0u;  // bit b: phase of accumulator buffer b
      bool ok = true;
      UnitInfo u;
      const uint32_t q_addr = smem_u32(S.q);
      for (int round = 0; ok && unit_at<kKind>(a, round, u); ++round) {
        if (!(ok = mbar_wait(&S.q_full, qi & 1, abort_flag, a.status, 20, budget))) break;
        ++qi;
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(128, u.nq * kHeads);
        for (int j = 0; j < u.ntiles; ++j) {
          if (!(ok = mbar_wait(&S.k_full[s], ph, abort_flag, a.status, 21, budget))) break;
          if (!(ok = mbar_wait(&S.t_empty[buf], ((tph >> buf) & 1u) ^ 1u, abort_flag, a.status, 22, budget))) break;
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
          tph ^= 1u << buf;
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
      mbar_wait_drain(&S.drain, 0, a.status, 23);
    }
  } else if (warp == kThreshWarp) {
    // ---------------- threshold warp ----------------
    // Raises each active row's threshold bin from its histogram, off the
    // epilogue's critical path, until every epilogue warpgroup is done.
    while (*(volatile int*)&S.epi_done < 4 && !*abort_flag) {
#pragma unroll 1
      for (int q = 0; q < kQB; ++q) tb_raise(S.rows[q], a.k, lane);
      __nanosleep(1000);
    }
  } else {
    // ---------------- epilogue: 16 warps in four warpgroups ----------------
    // A unit of nq queries gives each query a team of 4/nq warpgroups (one
    // for nq >= 3, the last warpgroup idle when nq == 3); team member m takes
    // the tiles jt with jt mod team == m (team is 1, 2 or 4), so the per-tile latency of a short
    // unit (decode, tails) overlaps across the team.  Per tile a warp waits
    // for its accumulator, pulls its 32 key rows x 64 heads out of TMEM,
    // frees the buffer, scores, and appends survivors of the threshold to its
    // own candidate segment; warps not on the tile only release it.  No
    // barrier inside the tile loop: the threshold warp raises the thresholds.
    const int slot = warp >> 2, lq = warp & 3, tid = threadIdx.x & 127;
    const uint32_t lane_base = (uint32_t)(lq * 32) << 16;
    const uint64_t pol_keep = l2_evict_last();  // candidate lists: kept in L2 until the row's select reads them
    uint32_t eph = 0u;  // bit b: phase of accumulator buffer b
    int buf = 0;
    UnitInfo u;
    bool ok = true;
    for (int round = 0; ok && unit_at<kKind>(a, round, u); ++round) {
      // team layout of this unit
      const int team = u.nq == 1 ? 4 : (u.nq == 2 ? 2 : 1);
      const int q = team == 1 ? slot : (team == 2 ? (slot & 1) : 0);
      const int member = team == 1 ? 0 : (team == 2 ? (slot >> 1) : slot);
      const bool active = q < u.nq;
      const int tbar = team == 1 ? 1 + slot : (team == 2 ? 5 + q : 7);
      const int tthr = 128 * team;
      const int ttid = member * 128 + tid;
      RowState& st = S.rows[q];
      const int nseg = 4 * team;
      const int64_t seg_stride = a.cand_cap / nseg;
      const int64_t row = (int64_t)u.row0 + q;
      // decode: a list per (row, slice), read later by the merge; else a
      // list per (CTA, query slot), reused by the CTA's next unit
      uint2* const cand0 = a.cand + (kKind == 1 ? (active ? row * a.splits + u.seq_split : 0)
                                                : (int64_t)blockIdx.x * kQB + q) * a.cand_cap;
      uint2* const my_seg = cand0 + (member * 4 + lq) * seg_stride;
      const ulonglong2* w2 = reinterpret_cast<const ulonglong2*>(S.w[q]);
      // per-unit scalars (kept in registers through the tile loop)
      // keys 0 .. pos are visible (pos = -1: none); positions fit in int (N <= INT_MAX)
      const int pos = active ? (int)slot_pos<kKind>(a, u, q) : -1;
      const unsigned n_vis = (unsigned)(pos + 1);
      const int ntiles = u.ntiles, nkeys = u.nkeys;
      const int key0 = u.tile0 * kTileKeys + lq * 32 + lane;
      const int32_t* kmap = (kKind == 2) ? a.key_map + (int64_t)u.seq_split * a.bank : (kKind == 4 ? a.key_map : nullptr);
      // fp8 keys: score = scale[key] * sum_h w ReLU(q . k8), scale > 0; decode
      // groups index the scales of their own sequence
      const float* kscale =
          !kScaled ? nullptr : ((kKind == 2 && a.k_off != nullptr) ? a.k_scale + a.k_off[u.seq_split] : a.k_scale);
      const int u_key_row0 = u.key_row0;
      if (active) {
        if (ttid == 0) tb_retire(st);
        named_bar(tbar, tthr);
        row_reset(st, ttid, tthr);
        if (ttid < kHeads) S.w[q][ttid] = 0.5f * a.w[row * kHeads + ttid];  // halved: see head_accumulate16
        named_bar(tbar, tthr);
        if (ttid == 0) tb_open(st);
      }
      int count = 0;  // my segment's fill
      // group refine: the bank slot -> key position of this warp's next tile,
      // loaded a whole tile ahead so its latency never sits on the tile's path
      int kp_next = -1;
      if (kKind == 2 && active && member < ntiles && key0 + member * kTileKeys < nkeys)
        kp_next = kmap[key0 + member * kTileKeys];
      ClusterWalk walk;
      if constexpr (kKind == 4) walk.start(a, u.row0);
      for (int jt = 0; jt < ntiles; ++jt) {
        if (!mbar_wait(&S.t_full[buf], (eph >> buf) & 1u, abort_flag, a.status, 30, budget)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const bool mine = active && (jt & (team - 1)) == member;
        const float thr = row_threshold(st);  // read early: its latency hides behind the tile's loads
        // +0.0f pairs
        std::conditional_t<kScaled, uint64_t[4], uint64_t> acc{};
        const uint32_t col = tmem_base + lane_base + (uint32_t)(buf * 256 + q * kHeads);
        if (mine) {
          if constexpr (!kScaled) {
            // the row's 64 columns in four loads of 16, each consumed before
            // the next: 16 registers for the row instead of 32
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float v[16];
              tmem_ld_32x32b_x16(col + 16 * c, v);
              tmem_ld_wait();
              if (c == 3) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.t_empty[buf]);
              }
              head_accumulate16(v, w2 + 4 * c, acc);
            }
          } else {
            float v[32];
            tmem_ld_32x32b_x32(col, v);
            tmem_ld_wait();
            head_accumulate32(v, w2, acc);
            tmem_ld_32x32b_x32(col + 32, v);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.t_empty[buf]);
            head_accumulate32(v, w2 + 8, acc);
          }
        } else {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.t_empty[buf]);
        }
        eph ^= 1u << buf;
        buf ^= 1;
        if (mine) {
          int key;  // local key index (inverted file: sorted key row)
          bool in_range;
          if constexpr (kKind == 4) {
            key = walk.row + lq * 32 + lane;
            in_range = key < walk.end;
          } else {
            key = key0 + (kKind == 3 ? routed_block(a, u, jt) : jt) * kTileKeys;
            in_range = key < nkeys;
          }
          int kpos = key;
          if constexpr (kKind == 2) {
            kpos = in_range ? kp_next : -1;
            const int nkey = key + team * kTileKeys;  // this warp's next tile
            kp_next = (nkey < nkeys && in_bounds(nkey < a.bank, a.status, 6)) ? kmap[nkey] : -1;
          } else if (kmap != nullptr) {
            kpos = in_range ? kmap[key] : -1;
          }
          float score = acc_sum(acc);
          if (kScaled && in_range) score *= kscale[kKind == 1 ? (int64_t)u_key_row0 + key : kpos];
          score = score + 0.0f;  // -0 -> +0
          const bool valid = in_range && (unsigned)kpos < n_vis;
          if (kDebug && valid) a.dbg_scores[row * a.dbg_ld + kpos] = score;
          row_append_seg(st, my_seg, count, score, (uint32_t)kpos, valid, thr, pol_keep, lane, seg_stride, a.status);
        }
        if constexpr (kKind == 4) walk.next(a);
      }
      if (!active) {
        ok = group_and(1 + slot, 128, ok);
        continue;
      }
      // the whole team agrees on success before any further barrier
      ok = group_and(tbar, tthr, ok);
      if (!ok) break;
      if constexpr (kKind == 1) {
        // decode: no selection here.  The slice's candidate list goes to the
        // merge with its segment counts and its bin histogram, so the key
        // stream pauses only for one short pass: an entry below the slice's
        // own exact threshold bin has k entries of the slice above it, so
        // it cannot be in the row's top k, and each warp drops those from
        // its segment (compacting in place) before the merge reads it.
        const int64_t o = row * a.splits + u.seq_split;
        if (ttid == 0) tb_close(st);
        named_bar(tbar, tthr);  // every append of the team has landed in the histogram
        if (ttid < 32) tb_finish(st, a.k, lane);
        named_bar(tbar, tthr);
        if (st.cge >= a.k) {
          const float keep_at = bin_floor(st.bstar);
          int kept = 0;
          for (int i0 = 0; i0 < count; i0 += 32 * 8) {
            uint2 e[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int i = i0 + j * 32 + lane;
              e[j] = i < count ? my_seg[i] : make_uint2(0u, 0u);
            }
            // every entry of this batch is in registers before any write,
            // and writes land below i0 + 256: no entry is lost
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const bool keep = (i0 + j * 32 + lane < count) && __uint_as_float(e[j].x) >= keep_at;
              const unsigned m = __ballot_sync(0xffffffffu, keep);
              if (keep) st_global_hint(my_seg + kept + __popc(m & lanemask_lt()), e[j], pol_keep);
              kept += __popc(m);
            }
          }
          count = kept;
        }
        if (lane == 0) a.out_cnt[o * kSegHdr + 1 + member * 4 + lq] = count;
        if (ttid == 0) a.out_cnt[o * kSegHdr] = nseg;
        for (int b = ttid; b < kBins; b += tthr) a.out_hist[o * kBins + b] = st.hist[b];
        named_bar(tbar, tthr);  // the histogram is read out before any member resets it
        continue;
      }
      if (lane == 0) st.seg_cnt[member * 4 + lq] = count;
      if (ttid == 0) tb_close(st);
      named_bar(tbar, tthr);
      if (ttid < 32) tb_finish(st, a.k, lane);
      named_bar(tbar, tthr);
      CandList cl;
      cl.base = cand0;
      cl.stride = seg_stride;
      cl.nseg = nseg;
      cl.cnt = st.seg_cnt;
      cl.l2 = false;
      row_select<8>(st, cl, a.k, row_out(a.out_idx + row * a.out_ld, a.out_val + row * a.out_ld, a.k, a.status),
                    S.stage[q], kStageCap, ttid, tthr, tbar, a.status);
    }
    if (tid == 0) atomicAdd(&S.epi_done, 1);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem_base, 512);
}

template <bool kDebug, int kKind, bool kScaled>
static int launch_tc(const CUtensorMap& tmQ, const CUtensorMap& tmK, const TcArgs& a, int grid, cudaStream_t stream) {
  // the shared-memory opt-in is a per-device function attribute: set it once
  // on each device the kernel runs on
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DSA_ERR_CUDA;
  const uint64_t bit = uint64_t(1) << dev;
  if (!(configured.load(std::memory_order_acquire) & bit)) {
    if (cudaFuncSetAttribute(tc_index_kernel<kDebug, kKind, kScaled>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kTcSmemBytes) != cudaSuccess)
      return DSA_ERR_CUDA;
    configured.fetch_or(bit, std::memory_order_release);
  }
  tc_index_kernel<kDebug, kKind, kScaled><<<grid, kTcThreads, kTcSmemBytes, stream>>>(tmQ, tmK, a);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// Failure-path controls set by dsa_debug_set_wait (process-wide).
static std::atomic<uint32_t> g_wait_us{0};
static std::atomic<int> g_hold_first_tile{0};

void set_wait_controls(uint32_t budget_us, int hold_first_tile) {
  g_wait_us.store(budget_us);
  g_hold_first_tile.store(hold_first_tile ? 1 : 0);
}

int launch_tc_index(const CUtensorMap& tmQ, const CUtensorMap& tmK, const TcArgs& args, int grid,
                    cudaStream_t stream) {
  static const char* const kNames[5] = {"dsa.score_topk.prefill", "dsa.score_topk.decode",
                                         "dsa.score_topk.group_refine", "dsa.score_topk.block_refine",
                                         "dsa.score_topk.ivf_refine"};
  const NvtxRange nvtx(args.kind >= 0 && args.kind <= 4 ? kNames[args.kind] : "dsa.score_topk");
  TcArgs a = args;
  a.wait_ns = (uint64_t)g_wait_us.load() * 1000u;
  a.hold_first_tile = g_hold_first_tile.load();
  if (a.kind < 0 || a.kind > 4 || (a.dbg_scores != nullptr && a.kind != 0)) return DSA_ERR_INVALID_ARG;
  const TimerSlot ts = timer_acquire();
  if (ts.start) cudaEventRecord(ts.start, stream);
  int r;
  const bool sc = a.k_scale != nullptr;
  if (a.dbg_scores != nullptr)
    r = sc ? launch_tc<true, 0, true>(tmQ, tmK, a, grid, stream) : launch_tc<true, 0, false>(tmQ, tmK, a, grid, stream);
  else if (a.kind == 0)
    r = sc ? launch_tc<false, 0, true>(tmQ, tmK, a, grid, stream) : launch_tc<false, 0, false>(tmQ, tmK, a, grid, stream);
  else if (a.kind == 1)
    r = sc ? launch_tc<false, 1, true>(tmQ, tmK, a, grid, stream) : launch_tc<false, 1, false>(tmQ, tmK, a, grid, stream);
  else if (a.kind == 2)
    r = sc ? launch_tc<false, 2, true>(tmQ, tmK, a, grid, stream) : launch_tc<false, 2, false>(tmQ, tmK, a, grid, stream);
  else if (a.kind == 3)
    r = sc ? launch_tc<false, 3, true>(tmQ, tmK, a, grid, stream) : launch_tc<false, 3, false>(tmQ, tmK, a, grid, stream);
  else
    r = sc ? launch_tc<false, 4, true>(tmQ, tmK, a, grid, stream) : launch_tc<false, 4, false>(tmQ, tmK, a, grid, stream);
  if (ts.end) cudaEventRecord(ts.end, stream);
  return r;
}

size_t tc_smem_bytes() { return kTcSmemBytes; }

}  // namespace dsa
