// dsa_topk.cuh — streaming per-query top-k over scores that never reach HBM.
//
// One RowState (shared memory) follows one query row while its keys stream
// past in tiles:
//   * a candidate list in global scratch (uint2 = {score bits, key index}),
//     with room for every key the row can see, so it can never overflow;
//   * a 1024-bin histogram of the appended scores (1/16-binade bins) and a
//     threshold bin b*: a score is appended only if its bin >= b*;
//   * after each tile one warp raises b* as far as "at least k appended
//     scores lie in bins above b*" still holds.  Every score that was ever
//     filtered out therefore has at least k scores strictly above it, so the
//     filter never drops a member of the exact top-k.
// At the end of the row, entries in bins > b* are all selected; the b* bin is
// resolved exactly by an MSD radix select (8-bit digits) on the 64-bit key
// (order-preserving score bits, then inverted key index), which realises the
// ranking "score descending, lower key index first" with no ties left.
#pragma once

#include "dsa_common.cuh"

namespace dsa {

struct RowState {
  uint32_t hist[kBins];
  int cnt;         // single-list path: entries appended
  int seg_cnt[16]; // segmented path: entries per segment (set at row end)
  int bstar;       // threshold bin
  int cge;         // appended entries whose bin >= bstar (exact at select time)
  int seen;        // single-list path: cnt at the last update
  int outpos;      // select: next output slot
  int stage_cnt;   // select: entries staged from the b* bin
  int dsel, above, hsel;  // select: radix step result
  int top;         // highest bin holding an appended entry
  uint32_t tb;     // tagged threshold (segmented path): gen << 17 | active << 16 | bstar
  int pad[1];
};

constexpr uint32_t kTbActive = 1u << 16;

// Candidate list: nseg segments; segment s starts at segp[s] (a table in
// shared memory) or, without a table, at base + s * stride; cnt[s] entries
// are used in segment s.
struct CandList {
  const uint2* __restrict__ base;
  int64_t stride;
  int nseg;
  const int* cnt;
  bool l2;  // entries written by other CTAs: read them through L2
  const uint2* const* segp = nullptr;
  uint64_t pol = 0;  // nonzero: the L2 policy of the reads (a final read lets the lines go)
  // counts may live in shared or global memory (written by other CTAs):
  // read them with volatile loads
  __device__ __forceinline__ int count(int s) const { return *(volatile const int*)(cnt + s); }
  __device__ __forceinline__ const uint2* seg(int s) const { return segp ? segp[s] : base + s * stride; }
  __device__ __forceinline__ uint2 load(const uint2* p) const {
    return pol ? ld_global_hint(p, pol) : (l2 ? __ldcg(p) : *p);
  }
  __device__ __forceinline__ int total() const {
    int n = 0;
    for (int s = 0; s < nseg; ++s) n += count(s);
    return n;
  }
  __device__ __forceinline__ uint2 at(int i) const {
    int s = 0;
    while (s + 1 < nseg && i >= count(s)) {
      i -= count(s);
      ++s;
    }
    return load(seg(s) + i);
  }
};

__device__ __forceinline__ void row_reset(RowState& st, int tid, int nthr) {
  for (int i = tid; i < kBins; i += nthr) st.hist[i] = 0u;
  if (tid == 0) {
    st.cnt = 0;
    st.bstar = 0;
    st.cge = 0;
    st.seen = 0;
    st.top = 0;
    for (int s = 0; s < 16; ++s) st.seg_cnt[s] = 0;
  }
}

// Called by all 32 lanes of one warp for one score per lane.
__device__ __forceinline__ void row_append(RowState& st, uint2* __restrict__ cand, float score,
                                           uint32_t key_out, bool valid, int lane, int64_t cap = 0,
                                           int* status = nullptr) {
  const int bin = score_bin(score);
  const bool pass = valid && (bin >= *(volatile int*)&st.bstar);
  const unsigned m = __ballot_sync(0xffffffffu, pass);
  if (m == 0u) return;
  int base = 0;
  if (lane == 0) base = atomicAdd(&st.cnt, __popc(m));
  base = __shfl_sync(0xffffffffu, base, 0);
  if (pass) {
    const int r = __popc(m & ((1u << lane) - 1u));
    if (in_bounds(base + r < cap, status, 1)) cand[base + r] = make_uint2(__float_as_uint(score), key_out);
    const unsigned mm = __match_any_sync(m, bin);
    if ((__ffs(mm) - 1) == lane) atomicAdd(&st.hist[bin], (uint32_t)__popc(mm));
  }
}

// The row's current threshold as a score bound (see bin_floor): read once
// per tile by each appending warp.  A stale read is a lower bound, which only
// lets more candidates through.
__device__ __forceinline__ float row_threshold(const RowState& st) {
  return bin_floor((int)(*(volatile const uint32_t*)&st.tb & 0xFFFFu));
}

// Appends to a warp-private segment: `count` (a register, warp-uniform) is
// the segment's fill; only the histogram and the top bin are shared.  `thr`
// is row_threshold(st): a score passes if it is at least the floor of the
// threshold bin, exactly as if its bin were compared; the bin itself is
// computed for passing scores only.  `pol`: the L2 policy of the stores (the
// list is read back once, at the row's end).  All 32 lanes call it.
__device__ __forceinline__ void row_append_seg(RowState& st, uint2* __restrict__ seg, int& count, float score,
                                               uint32_t key_out, bool valid, float thr, uint64_t pol, int lane,
                                               int64_t seg_cap = 0, int* status = nullptr) {
  const bool pass = valid && score >= thr;
  const unsigned m = __ballot_sync(0xffffffffu, pass);
  if (m != 0u) {  // warp-uniform: the warp's collectives stay outside any divergent region
    const int bin = score_bin(score);
    const int wmax = __reduce_max_sync(0xffffffffu, pass ? bin : -1);
    const int at = count + __popc(m & lanemask_lt());
    if (pass) {
      if (in_bounds(at < seg_cap, status, 2))
        st_global_hint(seg + at, make_uint2(__float_as_uint(score), key_out), pol);
      atomicAdd(&st.hist[bin], 1u);
    }
    // the top bin rises after the histogram: a raise reading an older top
    // only skips bins, which undercounts and stays safe
    if (lane == 0 && wmax > *(volatile int*)&st.top) atomicMax(&st.top, wmax);
    count += __popc(m);
  }
}

// Largest bin b in [b0, top] with sum_{b' >= b} hist[b'] >= k, reading the
// histogram once, top bin first (128 bins per step, 4 per lane).  Returns
// (b, that sum), or (-1, sum over [b0, top]) when fewer than k entries lie
// there.  Safe while other warps append: every value read is at most the
// bin's current count, so any sum it acts on undercounts.  All 32 lanes.
__device__ __forceinline__ int2 hist_scan(const RowState& st, int b0, int top, int k, int lane) {
  int S = 0;
  int found = -1, cge = 0;
  for (int hi = top; hi >= b0; hi -= 128) {
    int x[4];
    int t = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = hi - 4 * lane - j;
      x[j] = (i >= b0) ? (int)*(volatile const uint32_t*)&st.hist[i] : 0;
      t += x[j];
    }
    int p = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, p, o);
      if (lane >= o) p += y;
    }
    const int before = S + p - t;  // sum of the bins above this lane's four
    const unsigned m = __ballot_sync(0xffffffffu, S + p >= k);
    if (m) {
      const int l = __ffs(m) - 1;
      if (lane == l) {
        // the first of my four bins (highest first) where the running sum reaches k
        int c = before, f = -1, g = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          c += x[j];
          const bool hit = (f < 0) && (c >= k);
          f = hit ? hi - 4 * lane - j : f;
          g = hit ? c : g;
        }
        found = f;
        cge = g;
      }
      found = __shfl_sync(0xffffffffu, found, l);
      cge = __shfl_sync(0xffffffffu, cge, l);
      return make_int2(found, cge);
    }
    S += __shfl_sync(0xffffffffu, p, 31);
  }
  return make_int2(-1, S);
}

// Segmented path, unit start (one thread, then the caller zeroes the
// histogram and calls tb_open after a barrier): retag the threshold word with
// a new generation, inactive, so that no raise computed on the old row lands.
__device__ __forceinline__ void tb_retire(RowState& st) {
  const uint32_t gen = (*(volatile uint32_t*)&st.tb >> 17) + 1u;
  *(volatile uint32_t*)&st.tb = gen << 17;
  __threadfence_block();
}

__device__ __forceinline__ void tb_open(RowState& st) {
  __threadfence_block();
  *(volatile uint32_t*)&st.tb = (*(volatile uint32_t*)&st.tb & ~0xFFFFu) | kTbActive;
  __threadfence_block();
}

// Segmented path, row end (one thread, no appends in flight): stop raises.
__device__ __forceinline__ void tb_close(RowState& st) {
  atomicAnd(&st.tb, ~kTbActive);
  __threadfence_block();
}

// One pass of the threshold warp over a row: raise b* as far as the
// histogram allows, unless the row was retired or closed meanwhile.
__device__ __forceinline__ void tb_raise(RowState& st, int k, int lane) {
  const uint32_t t = *(volatile uint32_t*)&st.tb;
  if (!(t & kTbActive)) return;
  const int b0 = (int)(t & 0xFFFFu);
  const int top = *(volatile int*)&st.top;
  const int2 r = hist_scan(st, b0, top, k, lane);
  if (lane == 0 && r.x > b0) atomicCAS(&st.tb, t, (t & ~0xFFFFu) | (uint32_t)r.x);
  __syncwarp();
}

// Segmented path, row end after tb_close and a barrier: exact b* and cge for
// row_select.  All 32 lanes of one warp.
__device__ __forceinline__ void tb_finish(RowState& st, int k, int lane) {
  const int b0 = (int)(*(volatile uint32_t*)&st.tb & 0xFFFFu);
  const int top = *(volatile int*)&st.top;
  const int2 r = hist_scan(st, b0, top, k, lane);
  if (lane == 0) {
    st.bstar = r.x >= 0 ? r.x : b0;
    st.cge = r.y;
  }
  __syncwarp();
}

// Called by all 32 lanes of one warp while no appends to this row are in
// flight (between two barriers of the threads that append to it).
__device__ __forceinline__ void row_update(RowState& st, int k, int lane) {
  const int cnt = *(volatile int*)&st.cnt;
  int S = st.cge + (cnt - st.seen);  // every append since the last update has bin >= bstar
  int b = st.bstar;
  if (S - (int)st.hist[b] >= k) {
    for (;;) {
      const int i = b + lane;
      const int x = (i < kBins) ? (int)st.hist[i] : 0;
      int p = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, p, o);
        if (lane >= o) p += y;
      }
      // advancing past bin b+lane keeps S(b+lane+1) = S - p >= k
      const bool ok = (S - p >= k) && (i + 1 < kBins);
      const unsigned m = __ballot_sync(0xffffffffu, ok);
      const int n = __popc(m);
      if (n < 32) {
        const int pn = __shfl_sync(0xffffffffu, p, n > 0 ? n - 1 : 0);
        if (n > 0) S -= pn;
        b += n;
        break;
      }
      S -= __shfl_sync(0xffffffffu, p, 31);
      b += 32;
    }
  }
  __syncwarp();
  if (lane == 0) {
    st.bstar = b;
    st.cge = S;
    st.seen = cnt;
  }
  __syncwarp();
}

// One contiguous list whose length is *n (shared memory).
__device__ __forceinline__ CandList single_list(const uint2* base, const int* n) {
  CandList c;
  c.base = base;
  c.stride = 0;
  c.nseg = 1;
  c.cnt = n;
  c.l2 = false;
  return c;
}

struct BinSrc {
  CandList c;
  int bin;
  __device__ __forceinline__ bool get(int i, uint2& e) const {
    e = c.at(i);
    return score_bin(__uint_as_float(e.x)) == bin;
  }
};

// Where a row's selection goes: separate index / score arrays, or packed
// {score bits, index} pairs (partial lists that are merged later).
struct RowOut {
  int32_t* __restrict__ idx;
  float* __restrict__ val;
  uint2* __restrict__ pair;
  int k = 0;             // the row's slots (bounds checks of the debug build)
  int* status = nullptr;
  // outputs are written once and not read here again: streaming stores
  __device__ __forceinline__ void put(int p, uint2 e) const {
    if (!in_bounds((unsigned)p < (unsigned)k, status, 3)) return;
    if (pair != nullptr) {
      __stcs(pair + p, e);
    } else {
      __stcs(idx + p, (int32_t)e.y);
      __stcs(val + p, __uint_as_float(e.x));
    }
  }
  __device__ __forceinline__ void pad(int p) const {
    if (!in_bounds((unsigned)p < (unsigned)k, status, 4)) return;
    if (pair != nullptr) {
      __stcs(pair + p, make_uint2(0xff800000u, 0xffffffffu));
    } else {
      __stcs(idx + p, -1);
      __stcs(val + p, __int_as_float(0xff800000));
    }
  }
};

__device__ __forceinline__ RowOut row_out(int32_t* idx, float* val, int k, int* status) {
  return RowOut{idx, val, nullptr, k, status};
}
__device__ __forceinline__ RowOut pair_out(uint2* pair, int k, int* status) {
  return RowOut{nullptr, nullptr, pair, k, status};
}

__device__ __forceinline__ void emit(RowState& st, uint2 e, const RowOut& out) {
  const int p = atomicAdd(&st.outpos, 1);
  out.put(p, e);
}

// Warp 0 of a group: over a 256-bucket histogram h (bucket 255 ranks
// highest), the bucket dsel holding the remaining-th best entry, the count
// above it and the count in it, written to st.dsel / st.above / st.hsel.
__device__ __forceinline__ void pick_digit(const uint32_t* h, int remaining, RowState& st, int lane) {
  uint32_t c[8];
  uint32_t tot = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    c[j] = h[255 - 8 * lane - j];
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
        st.dsel = 255 - 8 * lane - j;
        st.above = (int)cum;
        st.hsel = (int)c[j];
        break;
      }
      cum += c[j];
    }
  }
}

// One MSD radix step over the entries of `src` that pass its filter and
// match (key & mask) == prefix: histogram of the 8-bit digit at `shift`,
// then the digit dsel holding the remaining-th best entry, the number of
// entries above it (above) and in it (hsel).  Group-wide (nthr threads,
// named barrier `bar`); st.hist is scratch.
template <class Src>
__device__ void radix_level(const Src& src, int n, uint64_t prefix, uint64_t mask, int shift, int remaining,
                            RowState& st, int tid, int nthr, int bar, int& dsel, int& above, int& hsel) {
  uint32_t* h = st.hist;
  for (int i = tid; i < 256; i += nthr) h[i] = 0u;
  named_bar(bar, nthr);
  for (int i = tid; i < n; i += nthr) {
    uint2 e;
    if (!src.get(i, e)) continue;
    const uint64_t key = sel_key(e);
    if ((key & mask) == prefix) atomicAdd(&h[(key >> shift) & 255u], 1u);
  }
  named_bar(bar, nthr);
  if (tid < 32) pick_digit(h, remaining, st, tid);
  named_bar(bar, nthr);
  dsel = st.dsel;
  above = st.above;
  hsel = st.hsel;
  named_bar(bar, nthr);
}

// Emits every entry of `src` (passing its filter) with (key & mask) >= prefix.
template <class Src>
__device__ void emit_at_least(const Src& src, int n, uint64_t prefix, uint64_t mask, RowState& st, const RowOut& out,
                              int tid, int nthr, int bar) {
  for (int i = tid; i < n; i += nthr) {
    uint2 e;
    if (!src.get(i, e)) continue;
    if ((sel_key(e) & mask) >= prefix) emit(st, e, out);
  }
  named_bar(bar, nthr);
}

// Warp-aggregated output: lanes with `sel` write their entry at
// consecutive output slots.  All 32 lanes of the warp call it.
__device__ __forceinline__ void emit_warp(RowState& st, bool sel, uint2 e, const RowOut& out, int lane) {
  const unsigned m = __ballot_sync(0xffffffffu, sel);
  if (m == 0u) return;
  int base = 0;
  if (lane == __ffs(m) - 1) base = atomicAdd(&st.outpos, __popc(m));
  base = __shfl_sync(0xffffffffu, base, __ffs(m) - 1);
  if (sel) {
    out.put(base + __popc(m & ((1u << lane) - 1u)), e);
  }
}

__device__ __forceinline__ int warp_excl_scan(int x, int lane, int& total) {
  int p = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, p, o);
    if (lane >= o) p += y;
  }
  total = __shfl_sync(0xffffffffu, p, 31);
  return p - x;
}

constexpr int kBatch = 8;

// Calls f(e, valid) for every entry of the list, kBatch independent loads in
// flight per thread.  The segments are dealt out to the group's warps (a warp
// streams whole segments), and every lane of a warp runs the same number of
// calls (valid = false past a segment's end), so f may use warp collectives.
template <class F>
__device__ __forceinline__ void for_each_cand(const CandList& c, int tid, int nthr, F&& f) {
  const int lane = tid & 31, warp = tid >> 5, nw = nthr >> 5;
  for (int s = warp; s < c.nseg; s += nw) {
    const uint2* seg = c.seg(s);
    const int n = c.count(s);
    for (int i0 = 0; i0 < n; i0 += 32 * kBatch) {
      uint2 e[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int i = i0 + j * 32 + lane;
        e[j] = (i < n) ? c.load(seg + i) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) f(e[j], i0 + j * 32 + lane < n);
    }
  }
}

// Classify outcomes as packed counter increments, so that one warp scan
// counts both: selected entries in the low 16 bits, staged ones in the high.
constexpr int kCatSel = 1, kCatStage = 1 << 16;

// Streams the candidate list in batches of kBatch entries per thread and
// classifies each entry with cls(e) -> 0 drop, kCatSel emit to the output,
// kCatStage stage into shared memory (entries beyond stage_cap are counted,
// not stored).
// Segments are dealt out to the group's warps; output and stage slots are
// taken with one warp scan and one atomic per warp and batch.  All nthr
// threads call it (nthr a multiple of 32).
template <class Cls>
__device__ __forceinline__ void classify_pass(const CandList& c, int tid, int nthr, RowState& st, const RowOut& out,
                                              uint2* stage, int stage_cap, Cls&& cls) {
  const int lane = tid & 31, warp = tid >> 5, nw = nthr >> 5;
  for (int s = warp; s < c.nseg; s += nw) {
    const uint2* seg = c.seg(s);
    const int n = c.count(s);
    for (int i0 = 0; i0 < n; i0 += 32 * kBatch) {
      uint2 e[kBatch];
      int cat[kBatch];
      int acc = 0;  // selected | staged << 16 (at most 8 of each a lane, 256 a warp)
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int i = i0 + j * 32 + lane;
        e[j] = (i < n) ? c.load(seg + i) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int i = i0 + j * 32 + lane;
        cat[j] = (i < n) ? cls(e[j]) : 0;
        acc += cat[j];
      }
      int tot;
      const int p = warp_excl_scan(acc, lane, tot);
      const int te = tot & 0xFFFF, ts = tot >> 16;
      int be = 0, bs = 0;
      if (lane == 0) {
        if (te) be = atomicAdd(&st.outpos, te);
        if (ts) bs = atomicAdd(&st.stage_cnt, ts);
      }
      be = __shfl_sync(0xffffffffu, be, 0) + (p & 0xFFFF);
      bs = __shfl_sync(0xffffffffu, bs, 0) + (p >> 16);
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        if (cat[j] == kCatSel) {
          out.put(be, e[j]);
          ++be;
        } else if (cat[j] == kCatStage) {
          if (bs < stage_cap) stage[bs] = e[j];
          ++bs;
        }
      }
    }
  }
}

__device__ __forceinline__ uint2 key_entry(uint64_t key) {
  const uint32_t o = (uint32_t)(key >> 32);
  const uint32_t u = (o & 0x80000000u) ? (o & 0x7fffffffu) : ~o;
  return make_uint2(u, ~(uint32_t)key);
}

// Emits the `need` best of the ns staged entries (need <= ns <= stage_cap,
// stage_cap <= kPer * nthr).  Entries move into registers (kPer a thread);
// MSD digit steps of 8 bits, starting at bit `shift` of the 64-bit key (bits
// above it are equal for all entries or already decided), drop or emit whole
// digit buckets until at most 128 entries remain undecided; those are ranked
// exactly by counting.  Group-wide (nthr threads, barrier `bar`).
template <int kResolvePerThread>
static __device__ __noinline__ void stage_resolve(RowState& st, uint2* stage, int ns, int need, int shift,
                                                  const RowOut out, int tid, int nthr, int bar) {
  const int lane = tid & 31;
  uint64_t key[kResolvePerThread];
  bool live[kResolvePerThread];
#pragma unroll
  for (int j = 0; j < kResolvePerThread; ++j) {
    const int i = j * nthr + tid;
    live[j] = i < ns;
    key[j] = live[j] ? sel_key(stage[i]) : 0ull;
  }
  int remaining = need, nlive = ns;
  uint32_t* h = st.hist;
  while (nlive > 128 && shift >= 0) {
    named_bar(bar, nthr);
    for (int i = tid; i < 256; i += nthr) h[i] = 0u;
    named_bar(bar, nthr);
#pragma unroll
    for (int j = 0; j < kResolvePerThread; ++j)
      if (live[j]) atomicAdd(&h[(key[j] >> shift) & 255u], 1u);
    named_bar(bar, nthr);
    if (tid < 32) pick_digit(h, remaining, st, tid);
    named_bar(bar, nthr);
    const int dsel = st.dsel, above = st.above, hsel = st.hsel;
#pragma unroll
    for (int j = 0; j < kResolvePerThread; ++j) {
      const int d = live[j] ? (int)((key[j] >> shift) & 255u) : -1;
      emit_warp(st, d > dsel, key_entry(key[j]), out, lane);
      live[j] = (d == dsel);
    }
    remaining -= above;
    nlive = hsel;
    shift -= 8;
  }
  // at most 128 undecided entries: compact them, rank each by counting
  named_bar(bar, nthr);
  if (tid == 0) st.stage_cnt = 0;
  named_bar(bar, nthr);
  uint64_t* kk = reinterpret_cast<uint64_t*>(stage);
#pragma unroll
  for (int j = 0; j < kResolvePerThread; ++j) {
    const unsigned m = __ballot_sync(0xffffffffu, live[j]);
    int base = 0;
    if (m && lane == __ffs(m) - 1) base = atomicAdd(&st.stage_cnt, __popc(m));
    base = __shfl_sync(0xffffffffu, base, m ? __ffs(m) - 1 : 0);
    if (live[j]) kk[base + __popc(m & ((1u << lane) - 1u))] = key[j];
  }
  named_bar(bar, nthr);
  for (int i = tid; i < nlive; i += nthr) {
    const uint64_t mine = kk[i];
    int rank = 0;
    for (int j = 0; j < nlive; ++j) rank += kk[j] > mine;
    if (rank < remaining) {
      const uint2 e = key_entry(mine);
      out.put(atomicAdd(&st.outpos, 1), e);
    }
  }
  named_bar(bar, nthr);
}

// First key bit below a threshold bin's resolution: inside bins 1..1022 all
// scores share sign, exponent and top 4 mantissa bits (key bits 63..51);
// the clamped end bins share nothing.
__device__ __forceinline__ int digit_shift_below(int bin) { return (bin > 0 && bin < kBins - 1) ? 43 : 56; }

// Final selection of one row: writes min(k, visible) entries to
// out[0..k) (any order), pads the rest with -1 / -inf, and
// returns the number of real entries.  Group-wide call (nthr threads, a
// multiple of 32, stage_cap <= kPer * nthr).  Expects st.bstar / st.cge
// exact (no appends in flight).
template <int kPer = 8>
static __device__ __noinline__ int row_select(RowState& st, const CandList cand, int k, const RowOut out,
                                              uint2* __restrict__ stage, int stage_cap, int tid, int nthr, int bar,
                                              int* status) {
  named_bar(bar, nthr);
  const int n = cand.total(), bstar = st.bstar, cge = st.cge;
  const int hb = (int)st.hist[bstar];
  named_bar(bar, nthr);
  if (tid == 0) {
    st.outpos = 0;
    st.stage_cnt = 0;
  }
  named_bar(bar, nthr);
  if (cge < k) {
    // b* never moved: every visible key was appended (n == cge < k)
    classify_pass(cand, tid, nthr, st, out, stage, 0, [](uint2) { return kCatSel; });
    named_bar(bar, nthr);
    for (int i = n + tid; i < k; i += nthr) out.pad(i);
    named_bar(bar, nthr);
    return n;
  }
  const int need = k - (cge - hb);
  // entries above the threshold bin are selected; the bin itself is staged
  // score_bin(f) > b*  <=>  f >= bin_floor(b* + 1) (none when b* is the top bin);
  // score_bin(f) == b* <=>  f >= bin_floor(b*) and not above
  const float f_hi = bstar >= kBins - 1 ? __int_as_float(0x7f800000) : bin_floor(bstar + 1), f_lo = bin_floor(bstar);
  classify_pass(cand, tid, nthr, st, out, stage, stage_cap, [f_hi, f_lo](uint2 e) {
    const float f = __uint_as_float(e.x);
    return f >= f_hi ? kCatSel : (f >= f_lo ? kCatStage : 0);
  });
  named_bar(bar, nthr);
  const int ns = st.stage_cnt;
  if (tid == 0 && (ns != hb || st.outpos != cge - hb)) report_error(status, DSA_ERR_INTERNAL, 1);
  if (ns <= stage_cap) {
    stage_resolve<kPer>(st, stage, ns, need, digit_shift_below(bstar), out, tid, nthr, bar);
    return k;
  }
  // The threshold bin holds more entries than the stage.  Inside bins
  // 1..1022 the score bits 18..11 order the bin: one counting pass picks the
  // sub-bucket holding the cut, one pass emits the sub-buckets above it and
  // stages the cut sub-bucket.
  if (bstar > 0 && bstar < kBins - 1) {
    uint32_t* h = st.hist;
    named_bar(bar, nthr);
    for (int i = tid; i < 256; i += nthr) h[i] = 0u;
    named_bar(bar, nthr);
    for_each_cand(cand, tid, nthr, [&](uint2 e, bool v) {
      if (v && score_bin(__uint_as_float(e.x)) == bstar) atomicAdd(&h[(e.x >> 11) & 255u], 1u);
    });
    named_bar(bar, nthr);
    if (tid < 32) pick_digit(h, need, st, tid);
    named_bar(bar, nthr);
    const int dsel = st.dsel, above = st.above, hsel = st.hsel;
    if (hsel <= stage_cap) {
      named_bar(bar, nthr);
      if (tid == 0) st.stage_cnt = 0;
      named_bar(bar, nthr);
      classify_pass(cand, tid, nthr, st, out, stage, stage_cap, [bstar, dsel](uint2 e) {
        if (score_bin(__uint_as_float(e.x)) != bstar) return 0;
        const int dg = (int)((e.x >> 11) & 255u);
        return dg > dsel ? kCatSel : (dg == dsel ? kCatStage : 0);
      });
      named_bar(bar, nthr);
      if (tid == 0 && (st.stage_cnt != hsel || st.outpos != cge - hb + above)) report_error(status, DSA_ERR_INTERNAL, 2);
      stage_resolve<kPer>(st, stage, hsel, need - above, 35, out, tid, nthr, bar);
      return k;
    }
    named_bar(bar, nthr);
    if (tid == 0) {
      st.outpos = cge - hb;  // nothing of the bin emitted yet
      st.stage_cnt = 0;
    }
    named_bar(bar, nthr);
  }
  // Still too many (massive ties): radix steps over the whole 64-bit key.
  const BinSrc gsrc{cand, bstar};
  const int n_all = n;
  uint64_t prefix = 0, mask = 0;
  int remaining = need;
  for (int shift = 56; shift >= 0; shift -= 8) {
    int dsel, above, hsel;
    radix_level(gsrc, n_all, prefix, mask, shift, remaining, st, tid, nthr, bar, dsel, above, hsel);
    remaining -= above;
    prefix |= (uint64_t)dsel << shift;
    mask |= (uint64_t)0xFFu << shift;
    if (hsel == remaining) break;
    if (hsel <= stage_cap) {
      if (tid == 0) st.stage_cnt = 0;
      named_bar(bar, nthr);
      for (int i = tid; i < n_all; i += nthr) {
        uint2 e;
        if (!gsrc.get(i, e)) continue;
        const uint64_t km = sel_key(e) & mask;
        if (km > prefix) {
          emit(st, e, out);
        } else if (km == prefix) {
          const int at = atomicAdd(&st.stage_cnt, 1);
          if (in_bounds(at < stage_cap, status, 5)) stage[at] = e;
        }
      }
      named_bar(bar, nthr);
      stage_resolve<kPer>(st, stage, hsel, remaining, shift - 8, out, tid, nthr, bar);
      return k;
    }
  }
  emit_at_least(gsrc, n_all, prefix, mask, st, out, tid, nthr, bar);
  return k;
}

}  // namespace dsa
