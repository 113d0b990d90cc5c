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
  int seg_cnt[4];  // segmented path: entries per segment (set at row end)
  int bstar;       // threshold bin
  int cge;         // appended entries whose bin >= bstar (exact at select time)
  int seen;        // single-list path: cnt at the last update
  int outpos;      // select: next output slot
  int stage_cnt;   // select: entries staged from the b* bin
  int dsel, above, hsel;  // select: radix step result
  int top;         // highest bin holding an appended entry
  int pad[2];
};

// Candidate list: nseg segments of `stride` entries each, cnt[s] used.
struct CandList {
  const uint2* base;
  int64_t stride;
  int nseg;
  int cnt[4];
  __device__ __forceinline__ int total() const {
    int n = 0;
    for (int s = 0; s < nseg; ++s) n += cnt[s];
    return n;
  }
  __device__ __forceinline__ uint2 at(int i) const {
    int s = 0;
    while (s + 1 < nseg && i >= cnt[s]) {
      i -= cnt[s];
      ++s;
    }
    return base[s * stride + i];
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
    for (int s = 0; s < 4; ++s) st.seg_cnt[s] = 0;
  }
}

// Called by all 32 lanes of one warp for one score per lane.
__device__ __forceinline__ void row_append(RowState& st, uint2* __restrict__ cand, float score,
                                           uint32_t key_out, bool valid, int lane) {
  const int bin = score_bin(score);
  const bool pass = valid && (bin >= *(volatile int*)&st.bstar);
  const unsigned m = __ballot_sync(0xffffffffu, pass);
  if (m == 0u) return;
  int base = 0;
  if (lane == 0) base = atomicAdd(&st.cnt, __popc(m));
  base = __shfl_sync(0xffffffffu, base, 0);
  if (pass) {
    const int r = __popc(m & ((1u << lane) - 1u));
    cand[base + r] = make_uint2(__float_as_uint(score), key_out);
    const unsigned mm = __match_any_sync(m, bin);
    if ((__ffs(mm) - 1) == lane) atomicAdd(&st.hist[bin], (uint32_t)__popc(mm));
  }
}

// Appends to a warp-private segment: `count` (a register, warp-uniform) is
// the segment's fill; only the histogram is shared.  All 32 lanes call it.
__device__ __forceinline__ void row_append_seg(RowState& st, uint2* __restrict__ seg, int& count, float score,
                                               uint32_t key_out, bool valid, int lane) {
  const int bin = score_bin(score);
  const bool pass = valid && (bin >= *(volatile int*)&st.bstar);
  const unsigned m = __ballot_sync(0xffffffffu, pass);
  if (m == 0u) return;
  if (pass) {
    seg[count + __popc(m & ((1u << lane) - 1u))] = make_uint2(__float_as_uint(score), key_out);
    const unsigned mm = __match_any_sync(m, bin);
    if ((__ffs(mm) - 1) == lane) atomicAdd(&st.hist[bin], (uint32_t)__popc(mm));
  }
  // highest occupied bin, raised after the histogram update; a raise that
  // reads an older value only skips bins, which undercounts and stays safe
  const int bmax = __reduce_max_sync(0xffffffffu, pass ? bin : 0);
  if (lane == 0 && bmax > *(volatile int*)&st.top) atomicMax(&st.top, bmax);
  count += __popc(m);
}

// Raises the threshold bin to the largest b with sum_{b' >= b} hist[b'] >= k,
// reading the histogram once, top bin first.  Safe while other warps append:
// every value read is at most the bin's current count, so the sum it acts on
// is never more than the true one.  With `exact` (no appends in flight) it
// also sets cge = that sum (or the total when fewer than k were appended).
// Called by all 32 lanes of one warp.
__device__ __forceinline__ void row_raise(RowState& st, int k, int lane, bool exact) {
  const int b0 = *(volatile int*)&st.bstar;
  const int top = *(volatile int*)&st.top;
  int S = 0;
  int found = -1, cge = 0;
  // 128 bins per step, 4 consecutive bins per lane, lane 0 highest
  for (int hi = top; hi >= b0; hi -= 128) {
    int x[4];
    int t = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = hi - 4 * lane - j;
      x[j] = (i >= b0) ? (int)*(volatile uint32_t*)&st.hist[i] : 0;
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
        int c = before;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          c += x[j];
          if (c >= k) {
            found = hi - 4 * lane - j;
            cge = c;
            break;
          }
        }
      }
      found = __shfl_sync(0xffffffffu, found, l);
      cge = __shfl_sync(0xffffffffu, cge, l);
      break;
    }
    S += __shfl_sync(0xffffffffu, p, 31);
  }
  __syncwarp();
  if (lane == 0) {
    if (found > b0) st.bstar = found;
    if (exact) st.cge = found >= 0 ? cge : S;
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

__device__ __forceinline__ CandList single_list(const uint2* base, int n) {
  CandList c;
  c.base = base;
  c.stride = 0;
  c.nseg = 1;
  c.cnt[0] = n;
  c.cnt[1] = c.cnt[2] = c.cnt[3] = 0;
  return c;
}

struct StageSrc {
  const uint2* p;
  __device__ __forceinline__ bool get(int i, uint2& e) const {
    e = p[i];
    return true;
  }
};

struct BinSrc {
  CandList c;
  int bin;
  __device__ __forceinline__ bool get(int i, uint2& e) const {
    e = c.at(i);
    return score_bin(__uint_as_float(e.x)) == bin;
  }
};

__device__ __forceinline__ void emit(RowState& st, uint2 e, int32_t* oidx, float* oval) {
  const int p = atomicAdd(&st.outpos, 1);
  oidx[p] = (int32_t)e.y;
  oval[p] = __uint_as_float(e.x);
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
  if (tid < 32) {
    const int lane = tid;
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
  named_bar(bar, nthr);
  dsel = st.dsel;
  above = st.above;
  hsel = st.hsel;
  named_bar(bar, nthr);
}

// Emits every entry of `src` (passing its filter) with (key & mask) >= prefix.
template <class Src>
__device__ void emit_at_least(const Src& src, int n, uint64_t prefix, uint64_t mask, RowState& st, int32_t* oidx,
                              float* oval, int tid, int nthr, int bar) {
  for (int i = tid; i < n; i += nthr) {
    uint2 e;
    if (!src.get(i, e)) continue;
    if ((sel_key(e) & mask) >= prefix) emit(st, e, oidx, oval);
  }
  named_bar(bar, nthr);
}

// Selects the `need` best entries (by sel_key) among the entries of `src`
// that pass its filter, and emits them.  All nthr threads of the group call
// it; the group synchronises on named barrier `bar`.
template <class Src>
__device__ void radix_emit(const Src& src, int n, int need, RowState& st, int32_t* oidx, float* oval, int tid,
                           int nthr, int bar) {
  uint64_t prefix = 0, mask = 0;
  int remaining = need;
  for (int shift = 56; shift >= 0; shift -= 8) {
    int dsel, above, hsel;
    radix_level(src, n, prefix, mask, shift, remaining, st, tid, nthr, bar, dsel, above, hsel);
    remaining -= above;
    prefix |= (uint64_t)dsel << shift;
    mask |= (uint64_t)0xFFu << shift;
    if (hsel == remaining) break;
  }
  emit_at_least(src, n, prefix, mask, st, oidx, oval, tid, nthr, bar);
}

// Final selection of one row: writes min(k, visible) entries to
// oidx[0..k), oval[0..k) (any order), pads the rest with -1 / -inf, and
// returns the number of real entries.  Group-wide call (nthr threads).
static __device__ __noinline__ int row_select(RowState& st, const CandList& cand, int k,
                                              int32_t* __restrict__ oidx, float* __restrict__ oval,
                                              uint2* __restrict__ stage, int stage_cap, int tid, int nthr, int bar,
                                              int* status) {
  named_bar(bar, nthr);
  const int n = cand.total(), bstar = st.bstar, cge = st.cge;
  named_bar(bar, nthr);
  if (tid == 0) {
    st.outpos = 0;
    st.stage_cnt = 0;
  }
  if (cge < k) {
    // b* never moved: every visible key was appended (n == cge < k)
    for (int i = tid; i < n; i += nthr) {
      const uint2 e = cand.at(i);
      oidx[i] = (int32_t)e.y;
      oval[i] = __uint_as_float(e.x);
    }
    for (int i = n + tid; i < k; i += nthr) {
      oidx[i] = -1;
      oval[i] = __int_as_float(0xff800000);
    }
    named_bar(bar, nthr);
    return n;
  }
  const int hb = (int)st.hist[bstar];
  const int need = k - (cge - hb);
  named_bar(bar, nthr);
  // entries above the threshold bin are selected; the bin itself is staged
  for (int i = tid; i < n; i += nthr) {
    const uint2 e = cand.at(i);
    const int b = score_bin(__uint_as_float(e.x));
    if (b > bstar) {
      emit(st, e, oidx, oval);
    } else if (b == bstar) {
      const int s = atomicAdd(&st.stage_cnt, 1);
      if (s < stage_cap) stage[s] = e;
    }
  }
  named_bar(bar, nthr);
  const int ns = st.stage_cnt;
  if (tid == 0 && (ns != hb || st.outpos != cge - hb)) report_error(status, DSA_ERR_INTERNAL, 1);
  if (ns <= stage_cap) {
    radix_emit(StageSrc{stage}, ns, need, st, oidx, oval, tid, nthr, bar);
    return k;
  }
  // The threshold bin holds more entries than the stage: narrow it with
  // radix steps over the candidate list until the selected sub-bucket fits.
  const BinSrc gsrc{cand, bstar};
  uint64_t prefix = 0, mask = 0;
  int remaining = need;
  for (int shift = 56; shift >= 0; shift -= 8) {
    int dsel, above, hsel;
    radix_level(gsrc, n, prefix, mask, shift, remaining, st, tid, nthr, bar, dsel, above, hsel);
    remaining -= above;
    prefix |= (uint64_t)dsel << shift;
    mask |= (uint64_t)0xFFu << shift;
    if (hsel == remaining) break;
    if (hsel <= stage_cap) {
      if (tid == 0) st.stage_cnt = 0;
      named_bar(bar, nthr);
      for (int i = tid; i < n; i += nthr) {
        uint2 e;
        if (!gsrc.get(i, e)) continue;
        const uint64_t km = sel_key(e) & mask;
        if (km > prefix) {
          emit(st, e, oidx, oval);
        } else if (km == prefix) {
          stage[atomicAdd(&st.stage_cnt, 1)] = e;
        }
      }
      named_bar(bar, nthr);
      radix_emit(StageSrc{stage}, hsel, remaining, st, oidx, oval, tid, nthr, bar);
      return k;
    }
  }
  emit_at_least(gsrc, n, prefix, mask, st, oidx, oval, tid, nthr, bar);
  return k;
}

}  // namespace dsa
