// Eviction decision, compaction of retained tokens, and decode-cache set-up.
//
// "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention
// and Contextualized Learnable Token Eviction": Fig. 2 caption (r_{j,h}
// decides whether a KV pair is evicted when it moves out of the sliding
// window; the attention sink is always kept) and Fig. 3 caption (the
// out-of-window cache segment has capped capacity and holds the sink and the
// LTE-retained KVs).
//
// compact_kernel: kCompactSplit CTAs per (batch, KV head) unit.  Each walks
// all of the unit's tokens in rounds of one thread per token (the mask is a
// few KiB): a warp ballot gives each retained token its rank inside the warp,
// a 32-entry scan over warp totals gives the warp offsets, and a running carry
// links the rounds.  This yields the ascending retained-position list idx, its
// length, and the inclusive prefix counts cnt; CTA part p writes the entries
// of its p-th share of the rounds.  Each CTA then copies the retained rows of
// those rounds (whose idx entries it wrote itself), and part 0 the sink rows,
// into a contiguous column segment with 16-byte vector loads, so the
// attention kernels read the "column" keys as dense tiles.  (Splitting a unit
// over several CTAs spreads the copy over more SMs than there are units.)
#include <math.h>

#include "lte_common.cuh"
#include "lte_internal.h"

namespace lte {

constexpr int kCompactThreads = 1024;
constexpr int kCompactSplit = 4;   // CTAs per unit
constexpr int kCompactPad = 64;    // zeroed slots after the retained rows (one key tile)

__device__ __forceinline__ void copy_row(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                         int nvec, int lane_in_row) {
  if (lane_in_row < nvec) dst[lane_in_row] = src[lane_in_row];
}

__global__ void __launch_bounds__(kCompactThreads)
compact_kernel(int T, int Hkv, int sink, int n_scored, float tau, const float* __restrict__ r,
               const uint8_t* __restrict__ mask, int32_t* __restrict__ idx,
               int32_t* __restrict__ nret, int32_t* __restrict__ cnt, const char* __restrict__ k,
               const char* __restrict__ v, Strides4 s, int elt, int D, char* __restrict__ k_col,
               char* __restrict__ v_col) {
  __shared__ int warp_tot[32];
  __shared__ int warp_off[32];
  __shared__ int round_total;
  const int u = blockIdx.x / kCompactSplit, part = blockIdx.x % kCompactSplit;
  const int b = u / Hkv, h = u % Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n_rounds = (T + kCompactThreads - 1) / kCompactThreads;
  const int r_lo = (int)((long long)n_rounds * part / kCompactSplit);
  const int r_hi = (int)((long long)n_rounds * (part + 1) / kCompactSplit);
  const long long row0 = (long long)u * T;
  const unsigned lt_mask = (1u << lane) - 1u;

  int carry = 0, own_lo = 0, own_hi = 0;                 // retained ordinals of this CTA's rounds
  constexpr int kAhead = 8;                              // rounds whose decisions load together
  bool mk[kAhead];
  for (int base = 0, rnd = 0; base < T; base += kCompactThreads, ++rnd) {
    if (rnd % kAhead == 0) {                             // this thread's next kAhead decisions
#pragma unroll
      for (int a = 0; a < kAhead; ++a) {
        const int jj = base + a * kCompactThreads + tid;
        mk[a] = false;
        if (jj < T && jj >= sink && jj < n_scored)
          mk[a] = mask ? (mask[row0 + jj] != 0) : (r[row0 + jj] >= tau);
      }
    }
    const bool mine = rnd >= r_lo && rnd < r_hi;          // rounds whose entries this CTA writes
    if (rnd == r_lo) own_lo = carry;
    const int j = base + tid;
    bool m = false;
#pragma unroll
    for (int a = 0; a < kAhead; ++a)
      if (a == rnd % kAhead) m = mk[a];
    const unsigned ballot = __ballot_sync(0xffffffffu, m);
    if (lane == 0) warp_tot[warp] = __popc(ballot);
    __syncthreads();
    if (warp == 0) {
      const int x = warp_tot[lane];
      int incl = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      warp_off[lane] = incl - x;
      if (lane == 31) round_total = incl;
    }
    __syncthreads();
    const int pos = carry + warp_off[warp] + __popc(ballot & lt_mask);
    if (mine && m) idx[row0 + pos] = j;
    if (mine && j < T) cnt[row0 + j] = pos + (m ? 1 : 0);
    carry += round_total;
    if (rnd == r_hi - 1) own_hi = carry;
    __syncthreads();
  }
  if (r_lo >= r_hi) own_lo = own_hi = carry;
  if (tid == 0 && part == 0) nret[u] = carry;
  if (k_col == nullptr) return;
  __syncthreads();   // this CTA's idx entries are visible to all of its threads

  // column segment: slot i < sink <- row i; slot sink + i <- row idx[i]
  const int nvec = D * elt / 16;
  const int rows_per_pass = kCompactThreads / nvec;
  const int rr = tid / nvec, lane_in_row = tid % nvec;
  const int nsink = (part == 0) ? (sink < T ? sink : T) : 0;
  const int total = nsink + (own_hi - own_lo);
  const long long col0 = (long long)u * (sink + T);
  // rows: the sinks (part 0), then retained ordinals [own_lo, own_hi)
  for (int i = rr; i < total; i += rows_per_pass) {
    const int o = own_lo + (i - nsink);
    const int j = (i < nsink) ? i : idx[row0 + o];
    const int slot = (i < nsink) ? i : sink + o;
    const long long src = ((long long)b * s.b + (long long)j * s.t + (long long)h * s.h) * elt;
    const long long dst = (col0 + slot) * D * elt;
    copy_row(reinterpret_cast<const uint4*>(k + src), reinterpret_cast<uint4*>(k_col + dst), nvec,
             lane_in_row);
    copy_row(reinterpret_cast<const uint4*>(v + src), reinterpret_cast<uint4*>(v_col + dst), nvec,
             lane_in_row);
  }
  // zero rows (part 3): the sink slots a short sequence leaves empty, [T, sink),
  // and the kCompactPad slots after the last retained row.  A 64-row tile the
  // attention kernels load from the segment then holds zeros, never stale
  // memory, past its valid rows: a masked key has P = 0, and 0 times a stale
  // NaN or Inf would still poison the output.
  if (part == kCompactSplit - 1) {
    const int z0 = sink + carry, z1 = min(sink + T, sink + carry + kCompactPad);
    const int e0 = T < sink ? T : sink, n_e = sink - e0;     // empty sink slots
    const int nz = n_e + (z1 > z0 ? z1 - z0 : 0);
    const uint4 zero = make_uint4(0, 0, 0, 0);
    for (int i = rr; i < nz; i += rows_per_pass) {
      const int slot = i < n_e ? e0 + i : z0 + (i - n_e);
      const long long dst = (col0 + slot) * D * elt;
      if (lane_in_row < nvec) {
        reinterpret_cast<uint4*>(k_col + dst)[lane_in_row] = zero;
        reinterpret_cast<uint4*>(v_col + dst)[lane_in_row] = zero;
      }
    }
  }
}

cudaError_t evict_compact(const lte_dims* d, const float* r, const uint8_t* mask, int n_scored,
                          int32_t* idx, int32_t* nret, int32_t* cnt, const void* k,
                          const void* v, Strides4 s, void* k_col, void* v_col,
                          cudaStream_t stream) {
  const int elt = d->dtype == LTE_BF16 ? 2 : 4;
  compact_kernel<<<d->B * d->Hkv * kCompactSplit, kCompactThreads, 0, stream>>>(
      d->T, d->Hkv, d->sink, n_scored, d->tau, r, mask, idx, nret, cnt, (const char*)k,
      (const char*)v, s, elt, d->D, (char*)k_col, (char*)v_col);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Lifetimes of retained tokens under the drop-the-lowest-score cap
// (LTE_CAP_LOWEST).  The segment after n arrivals holds the C best of them by
// (score, ordinal): a token is dropped -- possibly on arrival -- exactly when
// the C-th token that beats it has arrived.  So death[i] = max(i, j*) + 1,
// j* the ordinal at which the count of tokens beating i reaches C, scanning
// ordinals in order (T + 1 if it never does).
// One thread per ordinal, kLifeThreads ordinals per CTA; the unit's compacted
// scores pass through shared memory in tiles, read by every thread of the CTA
// at the same address (broadcast).  A CTA stops once all its threads have
// found their j*.
constexpr int kLifeThreads = 256;
constexpr int kLifeTile = 2048;

__global__ void __launch_bounds__(kLifeThreads)
lifetimes_kernel(int T, int cap, const float* __restrict__ r, const int32_t* __restrict__ idx,
                 const int32_t* __restrict__ nret, int32_t* __restrict__ death) {
  __shared__ float rc[kLifeTile];
  const int chunks = (T + kLifeThreads - 1) / kLifeThreads;
  const int u = blockIdx.x / chunks, tid = threadIdx.x;
  const long long row0 = (long long)u * T;
  const int n = nret[u];
  const int i0 = (blockIdx.x % chunks) * kLifeThreads;
  if (i0 >= n) return;
  const int i = i0 + tid;
  const bool valid = i < n;
  if (cap == 0 || n <= cap) {
    // C = 0: zero beaters suffice, every token is dropped on arrival (i + 1);
    // n <= C: at most n - 1 < C others, nobody is ever dropped
    if (valid) death[row0 + i] = cap == 0 ? i + 1 : T + 1;
    return;
  }
  const float ri = valid ? r[row0 + idx[row0 + i]] : 0.f;
  int beaten = 0, dies = T + 1;
  bool found = !valid;
  for (int j0 = 0; j0 < n; j0 += kLifeTile) {
    const int nj = min(kLifeTile, n - j0);
    __syncthreads();                                 // the previous tile has been read
    for (int jj = tid; jj < nj; jj += kLifeThreads) rc[jj] = r[row0 + idx[row0 + j0 + jj]];
    __syncthreads();
    if (!found) {
      for (int jj = 0; jj < nj; ++jj) {
        const int j = j0 + jj;
        const float x = rc[jj];
        beaten += (x > ri || (x == ri && j > i)) ? 1 : 0;   // j == i never counts
        if (beaten == cap) {
          dies = max(i, j) + 1;
          found = true;
          break;
        }
      }
    }
    if (__syncthreads_and(found)) break;
  }
  if (valid) death[row0 + i] = dies;
}

cudaError_t retained_lifetimes(const lte_dims* d, const float* r, const int32_t* idx,
                               const int32_t* nret, int32_t* death, cudaStream_t stream) {
  const long long ctas = (long long)((d->T + kLifeThreads - 1) / kLifeThreads) * d->B * d->Hkv;
  if (ctas > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  lifetimes_kernel<<<(unsigned)ctas, kLifeThreads, 0, stream>>>(d->T, d->cap, r, idx, nret, death);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Relaxed retention (training): the logit offset of every column-segment slot,
// log r / scale for the retained token in the slot (so that adding it to the
// raw score q.k multiplies the key's softmax weight by r), 0 for the sink
// slots, the empty slots and 64 padding floats at the end (the attention
// kernels read a whole 64-slot tile of offsets).  r is clamped below at 1e-30.
__global__ void __launch_bounds__(256)
slot_bias_kernel(long long n_slots, int T, int sink, float inv_scale, const float* __restrict__ r,
                 const int32_t* __restrict__ idx, const int32_t* __restrict__ nret,
                 float* __restrict__ bias) {
  const long long stride = (long long)sink + T;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n_slots + 64;
       e += (long long)gridDim.x * blockDim.x) {
    float b = 0.f;
    if (e < n_slots) {
      const long long u = e / stride;
      const int i = (int)(e - u * stride) - sink;
      if (i >= 0 && i < __ldg(nret + u)) {
        const int j = __ldg(idx + u * T + i);
        b = logf(fmaxf(__ldg(r + u * T + j), 1e-30f)) * inv_scale;
      }
    }
    bias[e] = b;
  }
}

size_t slot_bias_floats(const lte_dims* d) {
  return (size_t)d->B * d->Hkv * ((size_t)d->sink + d->T) + 64;
}

cudaError_t slot_bias(const lte_dims* d, const float* r, const int32_t* idx, const int32_t* nret,
                      float* bias, cudaStream_t stream) {
  const long long n_slots = (long long)d->B * d->Hkv * ((long long)d->sink + d->T);
  long long blocks = (n_slots + 64 + 255) / 256;
  blocks = blocks > 148 * 16 ? 148 * 16 : blocks;
  slot_bias_kernel<<<(unsigned)blocks, 256, 0, stream>>>(n_slots, d->T, d->sink, 1.0f / d->scale, r,
                                                         idx, nret, bias);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Decode-cache set-up from a prefilled prompt (Fig. 3 layout): window ring,
// sink slots, retained ring.  One CTA per unit.
__global__ void __launch_bounds__(256)
cache_init_kernel(int T, int Hkv, int D, int elt, int window, int sink, int cap, int cap_policy,
                  int T0, int n_scored, const char* __restrict__ k, const char* __restrict__ v,
                  Strides4 s, const float* __restrict__ r, const int32_t* __restrict__ idx,
                  const int32_t* __restrict__ cnt, const int32_t* __restrict__ death,
                  char* __restrict__ ck, char* __restrict__ cv, int32_t* __restrict__ pos,
                  float* __restrict__ win_r, int32_t* __restrict__ ret_total,
                  int32_t* __restrict__ meta, float* __restrict__ ret_r) {
  __shared__ int warp_tot[8];
  const int u = blockIdx.x, b = u / Hkv, h = u % Hkv, tid = threadIdx.x;
  const bool lowest = cap_policy == LTE_CAP_LOWEST;
  const int L = window + sink + cap;
  const long long row0 = (long long)u * T;
  const int last_out = T0 - 1 - window;                 // newest token outside the window
  // retained tokens the segment holds (all that left with a keep decision, or
  // under LTE_CAP_FIRST at most the first C), the i-th in ring slot i mod C
  const int n = last_out >= 0 ? held_retained(cnt[row0 + last_out], cap, cap_policy) : 0;
  const int ret_lo = (n - cap) > 0 ? n - cap : 0;

  // slot -> source token (or -1)
  for (int slot = tid; slot < L; slot += blockDim.x) {
    int j = -1;
    if (slot < window) {
      // newest token in this window slot, if it is inside (T0-1-w, T0-1]
      const int jj = T0 - 1 - ((T0 - 1 - slot) % window + window) % window;
      if (T0 > 0 && jj >= 0 && jj > last_out) j = jj;
      win_r[(long long)u * window + slot] = (j >= 0 && j < n_scored) ? r[row0 + j] : NAN;
    } else if (slot < window + sink) {
      const int jj = slot - window;
      if (jj <= last_out) j = jj;
    } else {
      const int rs = slot - window - sink;
      // retained ordinal i with i mod C == rs in [ret_lo, n) (LTE_CAP_LOWEST: below)
      if (n > 0 && !lowest) {
        int i = ret_lo + ((rs - ret_lo % cap) % cap + cap) % cap;
        if (i < n) j = idx[row0 + i];
      }
    }
    pos[(long long)u * L + slot] = j;
  }
  int held = n;
  if (lowest) {
    // the tokens held at count n, i < n with death[i] > n, in ordinal order in
    // slots 0, 1, ...: a ballot rank per warp plus the warp offsets, per round
    // of 256 ordinals
    const int lane = tid & 31, warp = tid >> 5;
    int carry = 0;
    for (int base = 0; base < n; base += 256) {
      const int i = base + tid;
      const bool keep = i < n && death[row0 + i] > n;
      const unsigned bal = __ballot_sync(0xffffffffu, keep);
      __syncthreads();                                // the previous round's totals are read
      if (lane == 0) warp_tot[warp] = __popc(bal);
      __syncthreads();
      int off = carry, tot = 0;
      for (int w = 0; w < 8; ++w) {
        if (w < warp) off += warp_tot[w];
        tot += warp_tot[w];
      }
      const int slot = off + __popc(bal & ((1u << lane) - 1u));
      if (keep && slot < cap) {
        const int j = idx[row0 + i];
        pos[(long long)u * L + window + sink + slot] = j;
        ret_r[(long long)u * cap + slot] = r[row0 + j];
      }
      carry += tot;
    }
    held = carry < cap ? carry : cap;
    for (int slot = held + tid; slot < cap; slot += blockDim.x)
      ret_r[(long long)u * cap + slot] = NAN;
  }
  __syncthreads();
  const int nvec = D * elt / 16;
  for (int i = tid; i < L * nvec; i += blockDim.x) {
    const int slot = i / nvec, c = i % nvec;
    const int j = pos[(long long)u * L + slot];
    if (j < 0) continue;
    const long long src = ((long long)b * s.b + (long long)j * s.t + (long long)h * s.h) * elt;
    const long long dst = ((long long)u * L + slot) * D * elt;
    reinterpret_cast<uint4*>(ck + dst)[c] = reinterpret_cast<const uint4*>(k + src)[c];
    reinterpret_cast<uint4*>(cv + dst)[c] = reinterpret_cast<const uint4*>(v + src)[c];
  }
  if (tid == 0) {
    ret_total[u] = held;
    if (u == 0) {
      meta[0] = T0;
      meta[1] = n_scored;
      meta[2] = n_scored;
      meta[3] = 0;
    }
  }
}

cudaError_t cache_init(const lte_dims* d, const lte_cache* c, const void* k, const void* v,
                       Strides4 s, const float* r, const int32_t* idx, const int32_t* cnt,
                       const int32_t* death, int T_prompt, int n_scored, cudaStream_t stream) {
  const int elt = d->dtype == LTE_BF16 ? 2 : 4;
  cache_init_kernel<<<d->B * d->Hkv, 256, 0, stream>>>(
      d->T, d->Hkv, d->D, elt, d->window, d->sink, d->cap, d->cap_policy, T_prompt, n_scored,
      (const char*)k, (const char*)v, s, r, idx, cnt, death, (char*)c->k, (char*)c->v, c->pos,
      c->win_r, c->ret_total, c->meta, c->ret_r);
  return cudaGetLastError();
}

}  // namespace lte
