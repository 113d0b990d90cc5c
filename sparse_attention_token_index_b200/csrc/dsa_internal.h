// dsa_internal.h — launch interfaces between the C ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

namespace dsa {

// An NVTX range around one kernel launch on the host, named for the step it
// runs, so that a profiler's timeline shows candidate scoring, selection,
// merging and the group steps apart (ADIndex — Deployment Guidance: profile
// the indexer's parts separately).  Costs a few nanoseconds without a tool.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Largest candidate bank of the group form: the bank ranking holds a whole
// bank in shared memory (8 bytes per key, 128 KB at this size).
constexpr int kMaxBank = 16384;

// Decode slices hand their raw candidate lists to the merge: per (row, slice)
// a header {nseg, count of segment 0 .. 15} and a kBins histogram; segment j
// of (row, slice) o starts at cand + o * cand_cap + j * (cand_cap / nseg).
constexpr int kSegHdr = 17;

// Arguments of the tensor-core kernel (see dsa_tc.cu).
//   kind 0: prefill rows.  Row r of Q sits at position
//           pos_base + min(r * pos_mul + pos_add, pos_clamp) and sees keys
//           0..pos (dense: pos_mul 1, pos_add 0; group proxies: pos_mul G,
//           pos_add G-1 so the proxy scans its group's last member's prefix).
//   kind 1: decode segments; unit v = (sequence v / splits, split v % splits);
//           each leaves its candidate list (no selection) for decode_merge.
//   kind 3: routed refine; unit v = query row v over its routed key blocks.
//   kind 2: group refine; unit v = (group v / mblocks, member block v % mblocks);
//           keys are the group's gathered bank rows, key_map gives their
//           positions.  With k_off / q_off set, group g is decode sequence g
//           (queries q_off[g].., at N_g - m_g + j; key_map local indices).
//   Decode units with q_off == nullptr have one query row per sequence
//   (row b: the proxies of a decode group scan).
struct TcArgs {
  int kind;
  const float* k_scale;     // per-key scale (fp8 keys), or null
  int n_rows;
  int n_units;
  int k;
  int64_t pos_base, pos_mul, pos_add, pos_clamp;
  const float* w;
  int32_t* out_idx;
  float* out_val;
  uint2* out_pair;   // decode (fp32 kernel): partial lists as {score bits, index} pairs
  int64_t out_ld;
  int* out_cnt;      // decode (tensor-core kernel): per (row, slice) segment header, kSegHdr ints
  uint32_t* out_hist;  // decode (tensor-core kernel): per (row, slice) bin histogram of its candidates
  uint2* cand;
  int64_t cand_cap;
  int* status;
  float* dbg_scores;
  int64_t dbg_ld;
  // decode
  const int64_t* k_off;
  const int32_t* q_off;
  int splits;
  int tiles_per_split;
  int64_t total_keys;     // rows of K: every k_off[b + 1] must stay within it
  const int* offsets_ok;  // decode groups: the call's device check of its offsets (null: none)
  // refine
  const int32_t* key_map;   // [ng, bank] bank key positions (-1 = empty)
  int bank;        // key slots per group in the gathered bank (its row stride)
  int group;
  int mblocks;
  int T;
  int key_slots;   // nonzero: every slot is streamed, key_map alone marks the valid ones
  // kind 0 rows see ((pos_base + r + 1) >> pos_shift) - 1 when pos_shift > 0
  // (the complete 128-key blocks before a query, for block routing)
  int pos_shift;
  // kind 3 (routed refine): one query row per unit; it streams the blocks
  // route_blocks[row, 0 .. min(route_n, complete blocks)) then its own
  // partial block, keys <= its position
  const int32_t* route_blocks;
  int route_n;
  // kind 4 (inverted-file refine): one query row per unit over its probed
  // clusters (route_blocks / route_n: cluster lists), whose keys sit at
  // sorted rows ivf_off[c] .. ivf_off[c+1]-1 (key_map: sorted row -> key);
  // ivf_tiles[row]: the tiles it streams
  const int32_t* ivf_off;
  const int32_t* ivf_tiles;
  int ivf_max_tiles;  // candidate lists hold this many tiles per query
  // failure-path controls (dsa_debug_set_wait; zero in normal calls): the
  // time budget of the waits between roles in ns (0 = the default), and a
  // first key tile that CTA 0's producer never loads, so that a wait runs out
  uint64_t wait_ns;
  int hold_first_tile;
};

// The current device, checked once: compute capability 10.0 (only sm_100a
// code is built) and its multiprocessor count.
int current_device(int* dev, int* sms);
// A driver entry point (resolved through the runtime, no libcuda link).
void* driver_entry(const char* name);
// 2-D bf16 tensor map over [rows, inner], box 64 x box_rows, 128-byte swizzle.
int make_map_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t inner, uint32_t box_rows);

// Event pair for timing one scoring-kernel launch (dsa_timer.cu); both null
// unless dsa_kernel_timer_start armed the timer and a slot is left.
struct TimerSlot {
  cudaEvent_t start = nullptr;
  cudaEvent_t end = nullptr;
};
TimerSlot timer_acquire();

int launch_tc_index(const CUtensorMap& tmQ, const CUtensorMap& tmK, const TcArgs& a, int grid,
                    cudaStream_t stream);
// dsa_debug_set_wait: time budget (microseconds) of the tensor-core kernel's
// inter-role waits (0 = default) and the held first tile of the failure-path test.
void set_wait_controls(uint32_t budget_us, int hold_first_tile);
size_t tc_smem_bytes();

// Exact fp32 CUDA-core path (any H <= 128, d <= 256, H*d <= 8192).
struct SimtArgs {
  int kind;          // 0 prefill rows, 1 decode (row task = (query row, split))
  int n_tasks;
  int H, d, k;
  int q_dtype, k_dtype;
  const void* Q;
  const float* w;
  const void* K;
  const float* K_scale;
  int64_t q_pos0;
  int32_t* out_idx;
  float* out_val;
  uint2* out_pair;   // decode: partial lists as {score bits, index} pairs
  int64_t out_ld;
  int* out_cnt;
  uint2* cand;
  int64_t cand_cap;
  int* status;
  float* dbg_scores;
  int64_t dbg_ld;
  const int64_t* k_off;
  const int32_t* q_off;
  int B;
  int splits;
  int keys_per_split;
  int64_t total_keys;     // rows of K: every k_off[b + 1] must stay within it
};
int launch_simt_index(const SimtArgs& a, int grid, cudaStream_t stream);
size_t simt_smem_bytes(int H, int d);

// Auxiliary kernels.
// Groups of G consecutive rows, or (seg given) rows seg[g] .. seg[g+1]-1 of
// nseg groups.
// `ok` (decode groups): the call's offsets check; the kernels that read device
// offsets do nothing when it failed.
int launch_proxy_mean(const void* Q, const float* w, int T, int H, int d, int G, int q_dtype, void* qbar,
                      float* wbar, cudaStream_t stream, const int32_t* seg = nullptr, int nseg = 0,
                      const int* ok = nullptr);
// rank_all: sort and write back the whole bank; otherwise only the top
// k + G - 1 entries are ranked (enough for Reuse) and the bank is not written.
// Refine with query-specific additions: map [ng, S] = bank (B) + own stretch (S - B).
// row_off (decode): bank indices are local to sequence g, whose rows start at row_off[g].
int launch_bank_gather(const void* K, int k_dtype, int d, const int32_t* bank, int ng, int bank_size,
                       void* Kg, cudaStream_t stream, const int64_t* row_off = nullptr, const int* ok = nullptr);
// Refine (prefill, bf16 keys with d = 128, bank_size <= 8192): map = the bank
// ordered by the proxy's score bin, highest first; Kg the matching key rows.
int launch_bank_order_gather(const void* K, const int32_t* bank_idx, const float* bank_val, int ng, int bank_size,
                             int32_t* map, void* Kg, cudaStream_t stream);
int launch_local_extend(const int32_t* bank, int ng, int B, int G, int T, int64_t q_pos0, const int32_t* q_off,
                        const int64_t* k_off, int S, int32_t* map, cudaStream_t stream, const int* ok = nullptr);
// q_off / k_off (decode): group g is sequence g with members q_off[g] ..
// q_off[g+1]-1 at positions N_g - m_g + j (local key indices).
int launch_bank_rank_reuse(int32_t* bank_idx, float* bank_val, int ng, int bank_size, int G, int T,
                           int64_t q_pos0, int k, int32_t* out_idx, float* out_val, int do_reuse, int rank_all,
                           cudaStream_t stream, const int32_t* q_off = nullptr, const int64_t* k_off = nullptr,
                           const int* ok = nullptr);
// parts [total_q, splits, k] {score bits, index} pairs, part_cnt [total_q, splits]
int launch_decode_merge(const uint2* parts, const int* part_cnt, int total_q, int splits, int k, int32_t* out_idx,
                        float* out_val, int* status, cudaStream_t stream, const int* ok = nullptr);
// The tensor-core decode scan's raw slice lists: cand [total_q, splits, cand_cap],
// hdr [total_q, splits, kSegHdr], hist [total_q, splits, kBins].
int launch_decode_merge_lists(const uint2* cand, int64_t cand_cap, const int* hdr, const uint32_t* hist, int total_q,
                              int splits, int k, int32_t* out_idx, float* out_val, int* status, cudaStream_t stream,
                              const int* ok = nullptr);
// Device check of decode offsets into the workspace header (offsets_ok + status word).
int launch_decode_offsets_check(const int64_t* k_off, const int32_t* q_off, int B, int64_t total_keys, int total_q,
                                int max_keys, void* workspace, cudaStream_t stream);
int launch_fill_scores(float* S, int64_t n, cudaStream_t stream);
// Block representatives of bf16 keys (fp8 keys widened; K_scale applied when given).
int launch_block_mean(const void* K, const float* K_scale, int64_t N, int d, void* R, cudaStream_t stream);
// Exact e4m3 -> bf16 copy of n bytes (n a multiple of 16, both 16-byte aligned).
int launch_e4m3_to_bf16(const uint8_t* src, int64_t n, void* dst, cudaStream_t stream);

// Inverted-file index (dsa_ivf.cu): views into the caller's index buffer.
struct IvfIndex {
  int32_t* off;     // [C+1] first sorted row of each cluster
  int32_t* perm;    // [N] sorted row -> key index
  int32_t* assign;  // [N] cluster of each key
  void* keys;       // [N, d] bf16, cluster after cluster
  void* cen_bf16;   // [C, d] bf16 centroids (routing)
  float* cen;       // [C, d] fp32 centroids
  size_t bytes;
};
IvfIndex ivf_index_view(void* base, int64_t N, int d, int C);
size_t ivf_build_scratch_bytes(int d, int C);
int ivf_build(const void* K, const float* K_scale, int64_t N, int d, int C, int iters, const IvfIndex& x,
              uint8_t* scratch, cudaStream_t st);
int launch_ivf_tiles(const int32_t* list, int n_probe, int T, const int32_t* off, int32_t* tiles, cudaStream_t st);

}  // namespace dsa
