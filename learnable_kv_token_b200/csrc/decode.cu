// Decode step of LTE: cache update + deferred batched scoring, then a
// persistent split-KV attention with an in-kernel log-sum-exp merge.
//
// "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention
// and Contextualized Learnable Token Eviction", Fig. 3 caption: the inference
// cache is a circular segment for in-window KVs plus an out-of-window segment
// of capped capacity for the retained KVs and the attention sink; scoring is
// batched and deferred as late as possible.  Fig. 2 caption: a KV pair is
// kept or evicted when it moves out of the window.  "Sparse Linear Attention:
// Viewing SWA from the Perspective of Linear Attention", section "Viewing SWA
// from the linear-state perspective": each new token overwrites one slot of
// the window (FIFO).
//
// Per step (both kernels read the step index t from meta[0] on the device, so
// the same two launches replay unchanged inside a CUDA graph):
//  1. decode_prep_kernel, one CTA per (batch, KV head) unit: token t-w leaves
//     its window slot (to its sink slot, into the retained ring, or dropped),
//     token t takes slot t mod w; then, when score_batch tokens are scorable,
//     the same CTA scores them from the window segment (score_tile, the same
//     arithmetic as lte_score).
//  2. decode_attn_kernel, persistent (about one CTA per SM): the valid slots
//     of all units form one flattened key space that is cut into equal
//     contiguous ranges, one per CTA.  A CTA streams its range in chunks of
//     64 keys: TMA copies (128B-swizzled) of the K, V and query rows into a
//     5-stage ring with bounded mbarrier waits; four warps take 16 keys each and run QK^T and PV on m16n8k16
//     bf16 MMAs (the G query heads of the group are MMA rows, so each K/V byte
//     is read once per group) with an online softmax.  At the end of each unit
//     the CTA writes an (m, l, o) partial; the last CTA of a unit (atomic
//     counter) merges the partials and writes o_t and lse_t; the last unit
//     advances meta.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "lte_common.cuh"
#include "lte_internal.h"
#include "score_cnn.cuh"
#include "score_tc.cuh"

namespace lte {

constexpr int kDecWarps = 4;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kDecChunk = 64;            // keys per pipeline stage
constexpr int kDecStages = 5;
constexpr int kDecMaxEntries = 256;      // chunk list entries per CTA
constexpr int kDecMaxParts = 8;          // CTAs sharing one unit

struct DecGeom {
  int n_ctas, per_cta, max_parts;
  bool single;             // one whole unit per CTA: no partials, no merge
};

static int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

static DecGeom dec_geom(const lte_dims* d) {
  const long long L = (long long)d->window + d->sink + d->cap;
  const long long W = (long long)d->B * d->Hkv * L;
  const long long want = (W + kDecChunk - 1) / kDecChunk;
  DecGeom g;
  const long long units = (long long)d->B * d->Hkv;
  if (units <= sm_count()) {
    // the units fit one wave: a CTA streams one whole unit and writes its
    // output itself (no split of a unit, hence no partials to merge)
    g.n_ctas = (int)units;
    g.per_cta = (int)L;
    g.max_parts = 1;
    g.single = true;
    return g;
  }
  g.n_ctas = (int)(want < sm_count() ? want : sm_count());
  if (g.n_ctas < 1) g.n_ctas = 1;
  g.per_cta = (int)((W + g.n_ctas - 1) / g.n_ctas);
  g.max_parts = (int)((L + g.per_cta - 1) / g.per_cta) + 1;
  g.single = false;
  return g;
}

// chunk-list bound for one CTA: range chunks + per-unit range splits and flushes
static bool dec_fits(const lte_dims* d) {
  const DecGeom g = dec_geom(d);
  const long long L = (long long)d->window + d->sink + d->cap;
  const long long units = (g.per_cta + L - 1) / L + 1;
  const long long rows = (long long)d->B * d->Hkv * L;          // TMA row coordinates are int32
  return (g.per_cta + kDecChunk - 1) / kDecChunk + 4 * units <= kDecMaxEntries &&
         g.max_parts <= kDecMaxParts &&
         rows < (1ll << 31) && (long long)d->B * d->Hq < (1ll << 31);
}

// workspace after the error word: partials [units][max_parts][G][D+4] fp32,
// then counters [units + 1] int32.
size_t decode_scratch_bytes(const lte_dims* d) {
  const size_t units = (size_t)d->B * d->Hkv;
  const size_t G = d->Hq / d->Hkv;
  return units * dec_geom(d).max_parts * G * (d->D + 4) * sizeof(float) +
         (units + 1) * sizeof(int32_t) + 64;
}

bool decode_supported(const lte_dims* d) { return dec_fits(d); }

// Programmatic dependent launch: a kernel may start while its predecessor in
// the stream finishes; griddepcontrol.wait blocks until the predecessor grid
// has completed and its memory is visible, launch_dependents lets the next
// kernel start its own prologue early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_next() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// The retained slot holding the lowest (score, position), over slots [0, cap)
// of one unit: each lane scans every 32nd slot, then a shuffle tree.  Called by
// a whole warp; every lane returns the same slot and score.
__device__ __forceinline__ int lowest_slot(const float* __restrict__ ret_r,
                                           const int32_t* __restrict__ ret_pos, int cap,
                                           float& r_min) {
  const int lane = threadIdx.x & 31;
  float br = INFINITY;
  int bp = 0x7fffffff, bs = -1;
  for (int i = lane; i < cap; i += 32) {
    const float x = ret_r[i];
    const int p = ret_pos[i];
    if (x < br || (x == br && p < bp)) br = x, bp = p, bs = i;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const float xr = __shfl_xor_sync(0xffffffffu, br, o);
    const int xp = __shfl_xor_sync(0xffffffffu, bp, o);
    const int xs = __shfl_xor_sync(0xffffffffu, bs, o);
    if (xr < br || (xr == br && xp < bp)) br = xr, bp = xp, bs = xs;
  }
  r_min = br;
  return bs;
}

// Where token `leaving` goes when it leaves the window (-1: dropped), and the
// retained count afterwards.  Called by a whole warp (LTE_CAP_LOWEST looks for
// the lowest held score when the segment is full); `held`/`r`/`rt` are read by
// every lane.  Under LTE_CAP_LOWEST the newcomer's score is written to its slot.
__device__ __forceinline__ int leaving_dst(int leaving, int held, float r, int rt, int window,
                                           int sink, int cap, int cap_policy, float tau,
                                           const int32_t* __restrict__ urow_pos,
                                           float* __restrict__ u_ret_r, DevError* err,
                                           int& rt_new) {
  const int lane = threadIdx.x & 31;
  rt_new = rt;
  if (leaving < 0) return -1;
  if (held != leaving) {
    if (lane == 0) record_error(err, LTE_ERR_DEVICE, kWhereDecodeIndex);
    return -1;
  }
  if (leaving < sink) return window + leaving;
  if (cap == 0 || !(r >= tau)) return -1;
  if (cap_policy == LTE_CAP_RECENT) {
    rt_new = rt + 1;
    return window + sink + rt % cap;
  }
  if (rt < cap) {                                 // FIRST and LOWEST fill slots in order
    rt_new = rt + 1;
    if (cap_policy == LTE_CAP_LOWEST && lane == 0) u_ret_r[rt] = r;
    return window + sink + rt;
  }
  if (cap_policy == LTE_CAP_FIRST) return -1;    // a full segment drops the newcomer
  float r_min;
  const int m = lowest_slot(u_ret_r, urow_pos + window + sink, cap, r_min);
  // the newcomer is the latest token, so it beats the lowest held one iff its
  // score is not below it
  if (m < 0 || r < r_min) return -1;
  __syncwarp();                                   // every lane has read the old score
  if (lane == 0) u_ret_r[m] = r;
  return window + sink + m;
}

// ---------------------------------------------------------------------------
struct PrepParams {
  int Hkv, D, elt, window, sink, cap, cap_policy, score_batch, future, n_units;
  float tau;
  const char* k_t;
  const char* v_t;
  char* ck;
  char* cv;
  int32_t* pos;
  float* win_r;
  int32_t* ret_total;
  int32_t* meta;
  int32_t* counters;
  DevError* err;
  float* ret_r;
};

template <typename T, bool kTc>
__global__ void __launch_bounds__(kTcThreads)
decode_prep_kernel(PrepParams pp, ScoreParams sp, RingKV<T> kv) {
  extern __shared__ __align__(128) float smem[];
  __shared__ int dst_sh;
  const int u = blockIdx.x, tid = threadIdx.x;
  const int L = pp.window + pp.sink + pp.cap;
  pdl_wait();              // the previous step's attention has finished with the cache
  pdl_launch_next();
  const int t = pp.meta[0];
  const int n_scored = pp.meta[1];
  const int leaving = t - pp.window;
  const int slot_w = t % pp.window;
  const long long urow = (long long)u * L;

  // ---- (1) cache update; every load is issued before any dependent store
  const int nvec = pp.D * pp.elt / 16;
  const long long wsrc = (urow + slot_w) * pp.D * pp.elt;
  uint4 kw, vw, kn, vn;
  if (tid < nvec) {
    kw = reinterpret_cast<const uint4*>(pp.ck + wsrc)[tid];      // leaving token (if any)
    vw = reinterpret_cast<const uint4*>(pp.cv + wsrc)[tid];
    kn = reinterpret_cast<const uint4*>(pp.k_t + (long long)u * pp.D * pp.elt)[tid];
    vn = reinterpret_cast<const uint4*>(pp.v_t + (long long)u * pp.D * pp.elt)[tid];
  }
  if (tid < 32) {
    int rt_new = 0, dst = -1;
    if (leaving >= 0) {
      const int held = pp.pos[urow + slot_w];
      const float r = pp.win_r[(long long)u * pp.window + slot_w];
      const int rt = pp.ret_total[u];
      dst = leaving_dst(leaving, held, r, rt, pp.window, pp.sink, pp.cap, pp.cap_policy, pp.tau,
                        pp.pos + urow, pp.ret_r + (long long)u * pp.cap, pp.err, rt_new);
      if (tid == 0 && rt_new != rt) pp.ret_total[u] = rt_new;
    }
    if (tid == 0) dst_sh = dst;
  }
  __syncthreads();
  const int dst_slot = dst_sh;
  if (tid < nvec) {
    if (dst_slot >= 0) {
      const long long dst = (urow + dst_slot) * pp.D * pp.elt;
      reinterpret_cast<uint4*>(pp.ck + dst)[tid] = kw;
      reinterpret_cast<uint4*>(pp.cv + dst)[tid] = vw;
    }
    reinterpret_cast<uint4*>(pp.ck + wsrc)[tid] = kn;
    reinterpret_cast<uint4*>(pp.cv + wsrc)[tid] = vn;
  }
  if (tid == 0) {
    if (dst_slot >= 0) pp.pos[urow + dst_slot] = leaving;
    pp.pos[urow + slot_w] = t;
    pp.win_r[(long long)u * pp.window + slot_w] = NAN;
    pp.counters[u] = 0;
    if (u == 0) pp.counters[pp.n_units] = 0;
  }
  __syncthreads();   // the new token is in the window for the scoring below

  // ---- (2) deferred batched scoring of the oldest scorable tokens
  const bool due = (t - pp.future) - n_scored + 1 >= pp.score_batch;
  if (u == 0 && tid == 0) pp.meta[2] = due ? n_scored + pp.score_batch : n_scored;
  if (!due) return;
  const int b = u / pp.Hkv, h = u % pp.Hkv;
  const int j_end = n_scored + pp.score_batch;
  for (int jb = n_scored; jb < j_end; jb += kScoreNT) {
    if constexpr (kTc)
      score_tile_tc<RingKV<T>>(sp, kv, b, h, jb, j_end, t + 1, reinterpret_cast<uint8_t*>(smem));
    else
      score_tile<T, RingKV<T>>(sp, kv, b, h, jb, j_end, t + 1, smem);
  }
}

// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32d(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void ldsm_x4d(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                         uint32_t& r3, bool trans) {
  if (trans)
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
  else
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16d(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16d(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
struct AttnParams {
  int Hq, Hkv, G, window, sink, cap, L, n_units, per_cta, max_parts, single;
  float scale_log2;
  const int32_t* ret_total;
  int32_t* meta;
  __nv_bfloat16* o_t;
  float* lse_t;
  float* part;
  int32_t* counters;
  DevError* err;
};

// 128B-swizzled tile written by TMA: [D/64 column halves][rows][128 bytes];
// byte offset of 16-byte chunk c of row r
__device__ __forceinline__ uint32_t sw128(int rows, int r, int c) {
  return (uint32_t)((c >> 3) * rows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}
__device__ __forceinline__ unsigned long long gtime_d() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool mbar_try_d(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait (1 s of global time); false when it ran out
__device__ __forceinline__ bool mbar_wait_d(uint32_t bar, uint32_t parity) {
  if (mbar_try_d(bar, parity)) return true;
  const unsigned long long t0 = gtime_d();
  while (!mbar_try_d(bar, parity))
    if (gtime_d() - t0 > 1000000000ull) return false;
  return true;
}
__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0,
                                       int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0,
                                       int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

template <int D>
__global__ void __launch_bounds__(kDecThreads, 1)
decode_attn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_q, const AttnParams p) {
  constexpr int KSTEPS = D / 16, DN = D / 8, HALVES = D / 64;
  constexpr int kKV = kDecChunk * D * 2;                  // K or V of one stage
  constexpr int kQ = 16 * D * 2;                          // Q rows of one stage
  constexpr int kStage = 2 * kKV + kQ;                    // multiple of 1 KiB
  extern __shared__ __align__(1024) uint8_t dsm[];
  float* o_sh = reinterpret_cast<float*>(dsm + kDecStages * kStage);    // [warps][16][D]
  float* m_sh = o_sh + kDecWarps * 16 * D;                               // [warps][16]
  float* l_sh = m_sh + kDecWarps * 16;                                   // [warps][16]
  int4* ents = reinterpret_cast<int4*>(l_sh + kDecWarps * 16);           // chunk list
  uint64_t* full = reinterpret_cast<uint64_t*>(ents + kDecMaxEntries);   // stage barriers
  int* n_ents = reinterpret_cast<int*>(full + kDecStages);
  int* is_last = n_ents + 1;
  int* t_sh = n_ents + 2;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((smem_u32d(dsm) & 1023u) != 0) {          // swizzle atoms need 1 KiB alignment
    if (tid == 0) record_error(p.err, LTE_ERR_DEVICE, 120);
    return;
  }
  pdl_launch_next();
  if (tid == 0) {
    for (int st = 0; st < kDecStages; ++st)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32d(full + st)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // meta[0] is not written by the preceding update kernel (only by the
  // attention grid of the previous step, which finished before that kernel
  // began).  Thread 0 reads it once for the CTA, then takes a ticket: the
  // CTA holding the last ticket advances meta at its end, when every CTA has
  // read the step index.
  int t = 0, ticket = 0;
  if (tid == 0) t = p.meta[0];
  pdl_wait();              // the cache update and scoring of this step are visible
  if (tid == 0)
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                 : "=r"(ticket)
                 : "l"(p.counters + p.n_units)
                 : "memory");
  if (tid == 0) *t_sh = t;
  __syncthreads();
  t = *t_sh;
  const int nw = min(p.window, t + 1);
  int ns = t - p.window + 1;
  ns = ns < 0 ? 0 : (ns > p.sink ? p.sink : ns);
  const long long W = (long long)p.n_units * p.L;
  const long long lo = (long long)blockIdx.x * p.per_cta;
  const long long hi = lo + p.per_cta < W ? lo + p.per_cta : W;

  // one elected thread issues the TMA copies of chunk i into stage i % kDecStages
  // (flush-only entries still load rows so that every stage use completes a phase)
  auto load = [&](int i) {
    const int4 e = ents[i];
    const uint32_t st = smem_u32d(dsm + (i % kDecStages) * kStage);
    const uint32_t bar = smem_u32d(full + i % kDecStages);
    const int b = e.x / p.Hkv, h = e.x % p.Hkv;
    const int row = e.x * p.L + e.y;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(kStage)
                 : "memory");
#pragma unroll
    for (int hf = 0; hf < HALVES; ++hf) {
      tma_2d(st + hf * kDecChunk * 128, &tm_k, bar, hf * 64, row);
      tma_2d(st + kKV + hf * kDecChunk * 128, &tm_v, bar, hf * 64, row);
      tma_2d(st + 2 * kKV + hf * 16 * 128, &tm_q, bar, hf * 64, b * p.Hq + h * p.G);
    }
  };

  // ---- chunk list: (unit, first slot, keys, last-of-unit) over the valid slots of [lo, hi).
  // The window chunks of the first unit need no retained count: their copies
  // start while the count loads.
  int issued = 0;
  if (tid == 0) {
    int n = 0;
    const int u_lo = (int)(lo / p.L), u_hi = (int)((hi - 1) / p.L);
    int rt[4];                                   // loads issued together, used below
#pragma unroll
    for (int k = 0; k < 4; ++k) rt[k] = (u_lo + k <= u_hi) ? p.ret_total[u_lo + k] : 0;
    for (int u = u_lo; u <= u_hi; ++u) {
      const int a = (int)((lo > (long long)u * p.L ? lo : (long long)u * p.L) - (long long)u * p.L);
      const long long ue = (long long)(u + 1) * p.L;
      const int bnd = (int)((hi < ue ? hi : ue) - (long long)u * p.L);
      const int rs[3] = {0, p.window, p.window + p.sink};
      const int first = n;
      for (int r = 0; r < 3; ++r) {
        const int re = r == 0 ? nw
                     : r == 1 ? p.window + ns
                              : p.window + p.sink +
                                    min(p.cap, u - u_lo < 4 ? rt[u - u_lo] : p.ret_total[u]);
        const int x = max(a, rs[r]), y = min(bnd, re);
        for (int s = x; s < y && n < kDecMaxEntries; s += kDecChunk)
          ents[n++] = make_int4(u, s, min(kDecChunk, y - s), 0);
        if (u == u_lo && r == 0)
          for (; issued < kDecStages - 1 && issued < n; ++issued) load(issued);
      }
      if (n == first && n < kDecMaxEntries) ents[n++] = make_int4(u, 0, 0, 0);   // flush only
      if (n > 0) ents[n - 1].w = 1;
    }
    *n_ents = n;
  }
  __syncthreads();
  const int n_ch = *n_ents;

  float o_acc[DN][4];
  float m_run[2], l_run[2];
  auto reset = [&]() {
#pragma unroll
    for (int i = 0; i < DN; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) o_acc[i][e] = 0.f;
    m_run[0] = m_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.f;
  };
  reset();

  if (tid == 0)
    for (; issued < kDecStages - 1 && issued < n_ch; ++issued) load(issued);
  int i = 0;
#pragma unroll 1
  for (; i < n_ch; ++i) {
    if (tid == 0 && i + kDecStages - 1 < n_ch) load(issued++);
    const bool ok = mbar_wait_d(smem_u32d(full + i % kDecStages), (i / kDecStages) & 1);
    if (__syncthreads_or(!ok)) {
      if (tid == 0) record_error(p.err, LTE_ERR_TIMEOUT, 121);
      break;
    }
    const int4 e = ents[i];
    const uint8_t* st = dsm + (i % kDecStages) * kStage;
    const int k0 = warp * 16;                 // this warp's 16 keys of the chunk
    if (k0 < e.z) {
      uint32_t qf[KSTEPS][4];
#pragma unroll
      for (int kst = 0; kst < KSTEPS; ++kst) {
        const int r = lane & 15, c = kst * 2 + (lane >> 4);
        ldsm_x4d(smem_u32d(st + 2 * kKV + sw128(16, r, c)), qf[kst][0], qf[kst][1], qf[kst][2],
                 qf[kst][3], false);
      }
      float s[2][4] = {};
#pragma unroll
      for (int kst = 0; kst < KSTEPS; ++kst) {
        const int r = k0 + ((lane >> 4) << 3) + (lane & 7);
        const int c = kst * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4d(smem_u32d(st + sw128(kDecChunk, r, c)), b0, b1, b2, b3, false);
        mma_bf16d(s[0], qf[kst], b0, b1);
        mma_bf16d(s[1], qf[kst], b2, b3);
      }
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int key = k0 + nt * 8 + ((lane & 3) << 1) + (q & 1);
          s[nt][q] = key < e.z ? s[nt][q] * p.scale_log2 : -INFINITY;
          mx[q >> 1] = fmaxf(mx[q >> 1], s[nt][q]);
        }
      float corr[2], mu[2];
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 1));
        mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 2));
        const float m_new = fmaxf(m_run[hr], mx[hr]);
        mu[hr] = m_new == -INFINITY ? 0.f : m_new;
        corr[hr] = m_run[hr] == -INFINITY ? 0.f : exp2f(m_run[hr] - mu[hr]);
        m_run[hr] = m_new;
        l_run[hr] *= corr[hr];
      }
      uint32_t pf[4];
      {
        float pv[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            pv[nt][q] = exp2f(s[nt][q] - mu[q >> 1]);
            l_run[q >> 1] += pv[nt][q];
          }
        pf[0] = pack_bf16d(pv[0][0], pv[0][1]);
        pf[1] = pack_bf16d(pv[0][2], pv[0][3]);
        pf[2] = pack_bf16d(pv[1][0], pv[1][1]);
        pf[3] = pack_bf16d(pv[1][2], pv[1][3]);
      }
#pragma unroll
      for (int i2 = 0; i2 < DN; ++i2) {
        o_acc[i2][0] *= corr[0]; o_acc[i2][1] *= corr[0];
        o_acc[i2][2] *= corr[1]; o_acc[i2][3] *= corr[1];
      }
#pragma unroll
      for (int dp = 0; dp < DN / 2; ++dp) {
        const int r = k0 + (((lane >> 3) & 1) << 3) + (lane & 7);
        const int c = dp * 2 + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4d(smem_u32d(st + kKV + sw128(kDecChunk, r, c)), b0, b1, b2, b3, true);
        mma_bf16d(o_acc[2 * dp], pf, b0, b1);
        mma_bf16d(o_acc[2 * dp + 1], pf, b2, b3);
      }
    }
    if (e.w) {
      // ---- end of this CTA's part of unit e.x: merge the warps, publish the partial
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        l_run[hr] += __shfl_xor_sync(0xffffffffu, l_run[hr], 1);
        l_run[hr] += __shfl_xor_sync(0xffffffffu, l_run[hr], 2);
        const int r = (lane >> 2) + hr * 8;
        if ((lane & 3) == 0) {
          m_sh[warp * 16 + r] = m_run[hr];
          l_sh[warp * 16 + r] = l_run[hr];
        }
#pragma unroll
        for (int i2 = 0; i2 < DN; ++i2) {
          const int dcol = i2 * 8 + ((lane & 3) << 1);
          o_sh[(warp * 16 + r) * D + dcol] = o_acc[i2][hr * 2];
          o_sh[(warp * 16 + r) * D + dcol + 1] = o_acc[i2][hr * 2 + 1];
        }
      }
      __syncthreads();
      const int u = e.x;
      if (p.single) {
        // the CTA holds the whole unit: combine its warps and write o_t, lse_t
        const int b = u / p.Hkv, h = u % p.Hkv;
        for (int i2 = tid; i2 < p.G * (D / 4); i2 += kDecThreads) {
          const int g = i2 / (D / 4), d4 = (i2 % (D / 4)) * 4;
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, m_sh[w * 16 + g]);
          float l = 0.f;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int w = 0; w < kDecWarps; ++w) {
            const float mw = m_sh[w * 16 + g];
            const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
            l += l_sh[w * 16 + g] * f;
            const float4 ow = *reinterpret_cast<const float4*>(o_sh + (w * 16 + g) * D + d4);
            acc.x += ow.x * f; acc.y += ow.y * f; acc.z += ow.z * f; acc.w += ow.w * f;
          }
          const float inv = 1.f / l;
          __nv_bfloat16* orow = p.o_t + ((long long)b * p.Hq + h * p.G + g) * D + d4;
          *reinterpret_cast<uint2*>(orow) =
              make_uint2(pack_bf16d(acc.x * inv, acc.y * inv), pack_bf16d(acc.z * inv, acc.w * inv));
          if (d4 == 0 && p.lse_t != nullptr)
            p.lse_t[(long long)b * p.Hq + h * p.G + g] = (M + log2f(l)) * 0.69314718055994531f;
        }
        reset();
        __syncthreads();   // stage i % kDecStages and the merge buffers are free again
        continue;
      }
      const int c_first = (int)(((long long)u * p.L) / p.per_cta);
      const int c_last = (int)(((long long)u * p.L + p.L - 1) / p.per_cta);
      const int n_parts = c_last - c_first + 1;
      // partial layout per (unit, part): [G][D + 4] fp32 = {m, l, pad, pad, o[D]}
      float* up = p.part + (long long)u * p.max_parts * p.G * (D + 4);
      float* mine = up + (long long)(blockIdx.x - c_first) * p.G * (D + 4);
      for (int i2 = tid; i2 < p.G * (D / 4); i2 += kDecThreads) {
        const int g = i2 / (D / 4), d4 = (i2 % (D / 4)) * 4;
        float M = -INFINITY;
        float f[kDecWarps];
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, m_sh[w * 16 + g]);
        float l = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
          const float mw = m_sh[w * 16 + g];
          f[w] = mw == -INFINITY ? 0.f : exp2f(mw - M);
          l += l_sh[w * 16 + g] * f[w];
        }
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
          const float4 ow = *reinterpret_cast<const float4*>(o_sh + (w * 16 + g) * D + d4);
          acc.x += ow.x * f[w]; acc.y += ow.y * f[w]; acc.z += ow.z * f[w]; acc.w += ow.w * f[w];
        }
        *reinterpret_cast<float4*>(mine + g * (D + 4) + 4 + d4) = acc;
        if (d4 == 0) *reinterpret_cast<float4*>(mine + g * (D + 4)) = make_float4(M, l, 0.f, 0.f);
      }
      __threadfence();
      __syncthreads();
      if (tid == 0) *is_last = atomicAdd(&p.counters[u], 1) == n_parts - 1;
      __syncthreads();
      if (*is_last) {
        __threadfence();
        const int b = u / p.Hkv, h = u % p.Hkv;
        for (int i2 = tid; i2 < p.G * (D / 4); i2 += kDecThreads) {
          const int g = i2 / (D / 4), d4 = (i2 % (D / 4)) * 4;
          float4 ml[kDecMaxParts], ov[kDecMaxParts];
#pragma unroll
          for (int sp = 0; sp < kDecMaxParts; ++sp)       // every load issued before any use
            if (sp < n_parts) {
              const float* pp = up + (sp * p.G + g) * (D + 4);
              ml[sp] = __ldcg(reinterpret_cast<const float4*>(pp));
              ov[sp] = __ldcg(reinterpret_cast<const float4*>(pp + 4 + d4));
            }
          float M = -INFINITY;
#pragma unroll
          for (int sp = 0; sp < kDecMaxParts; ++sp) if (sp < n_parts) M = fmaxf(M, ml[sp].x);
          float l = 0.f;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int sp = 0; sp < kDecMaxParts; ++sp)
            if (sp < n_parts && ml[sp].x != -INFINITY) {
              const float fw = exp2f(ml[sp].x - M);
              l += ml[sp].y * fw;
              acc.x += ov[sp].x * fw; acc.y += ov[sp].y * fw;
              acc.z += ov[sp].z * fw; acc.w += ov[sp].w * fw;
            }
          const float inv = 1.f / l;
          __nv_bfloat16* orow = p.o_t + ((long long)b * p.Hq + h * p.G + g) * D + d4;
          *reinterpret_cast<uint2*>(orow) =
              make_uint2(pack_bf16d(acc.x * inv, acc.y * inv), pack_bf16d(acc.z * inv, acc.w * inv));
          if (d4 == 0 && p.lse_t != nullptr)
            p.lse_t[(long long)b * p.Hq + h * p.G + g] = (M + log2f(l)) * 0.69314718055994531f;
        }
      }
      reset();
    }
    __syncthreads();     // stage i % kDecStages and the merge buffers are free again
  }
  // copies issued but not consumed (only after a wait ran out) land before exit
  if (tid == 0)
    for (int j = i; j < issued; ++j) mbar_wait_d(smem_u32d(full + j % kDecStages), (j / kDecStages) & 1);
  // every CTA has read the step index before taking its ticket: the last one advances it
  if (tid == 0 && ticket == (int)gridDim.x - 1) {
    p.meta[0] = t + 1;
    p.meta[1] = p.meta[2];
  }
}

// launch with programmatic stream serialization (see pdl_wait)
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <typename T>
static cudaError_t launch_prep(const lte_dims* d, const lte_cnn* cnn, const lte_cache* c,
                               const void* k_t, const void* v_t, int score_batch,
                               int32_t* counters, DevError* err, cudaStream_t stream) {
  PrepParams pp{};
  pp.Hkv = d->Hkv; pp.D = d->D; pp.elt = sizeof(T); pp.window = d->window; pp.sink = d->sink;
  pp.cap = d->cap; pp.cap_policy = d->cap_policy; pp.score_batch = score_batch;
  pp.future = (cnn->k1 - 1 - cnn->past1) + (cnn->k2 - 1 - cnn->past2);
  pp.n_units = d->B * d->Hkv; pp.tau = d->tau;
  pp.k_t = (const char*)k_t; pp.v_t = (const char*)v_t;
  pp.ck = (char*)c->k; pp.cv = (char*)c->v; pp.pos = c->pos; pp.win_r = c->win_r;
  pp.ret_total = c->ret_total; pp.meta = c->meta; pp.counters = counters; pp.err = err;
  pp.ret_r = c->ret_r;
  ScoreParams sp = score_params(d, cnn);
  sp.window = d->window;
  sp.win_r = c->win_r;
  const int L = d->window + d->sink + d->cap;
  RingKV<T> kv{(const T*)c->k, (const T*)c->v, d->Hkv, L, d->window, d->D};
  // the same scoring tile as lte_score for this shape, so decode scores equal prefill scores
  if (score_tc_supported(cnn->c_hid, cnn->k1, cnn->k2)) {
    const size_t smem = score_tc_smem_bytes(d->D, cnn->c_hid, cnn->k2);
    cudaError_t e = cudaFuncSetAttribute(decode_prep_kernel<T, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(decode_prep_kernel<T, true>, dim3(pp.n_units), dim3(kTcThreads), smem, stream,
                      pp, sp, kv);
  }
  const size_t smem = sizeof(float) * score_smem_floats(d->D, cnn->c_hid, cnn->k1, cnn->k2);
  cudaError_t e = cudaFuncSetAttribute(decode_prep_kernel<T, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_prep_kernel<T, false>, dim3(pp.n_units), dim3(kScoreThreads), smem,
                    stream, pp, sp, kv);
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// 2-D bf16 tensor map over `rows` rows of D elements, boxes of 64 x box_rows, 128B swizzle
static bool rows_map(CUtensorMap* m, const void* base, long long rows, int D, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 tensor map over `rows` rows of D elements seen as (64 columns, row,
// D/64 column halves): one box of 64 x box_rows x D/64 lands as [half][row][128 B],
// 128B-swizzled -- the layout of D/64 separate 2-D boxes, in one copy.
static bool rows_map_halves(CUtensorMap* m, const void* base, long long rows, int D, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)(D / 64)};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, 128};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, (cuuint32_t)(D / 64)};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
static cudaError_t launch_attn(const lte_dims* d, const lte_cache* c, const void* q_t, void* o_t,
                               float* lse_t, float* part, int32_t* counters, DevError* err,
                               cudaStream_t stream) {
  const DecGeom g = dec_geom(d);
  AttnParams p{};
  p.Hq = d->Hq; p.Hkv = d->Hkv; p.G = d->Hq / d->Hkv; p.window = d->window; p.sink = d->sink;
  p.cap = d->cap; p.L = d->window + d->sink + d->cap; p.n_units = d->B * d->Hkv;
  p.per_cta = g.per_cta; p.max_parts = g.max_parts; p.single = g.single ? 1 : 0;
  p.scale_log2 = d->scale * 1.4426950408889634f;
  p.ret_total = c->ret_total; p.meta = c->meta;
  p.o_t = (__nv_bfloat16*)o_t; p.lse_t = lse_t; p.part = part; p.counters = counters; p.err = err;
  CUtensorMap mk, mv, mq;
  const long long rows = (long long)p.n_units * p.L;
  if (!rows_map(&mk, c->k, rows, D, kDecChunk) || !rows_map(&mv, c->v, rows, D, kDecChunk) ||
      !rows_map(&mq, q_t, (long long)d->B * d->Hq, D, 16))
    return cudaErrorInvalidValue;
  const size_t stage = 2 * (size_t)kDecChunk * D * 2 + 16 * D * 2;
  const size_t smem = kDecStages * stage + (size_t)kDecWarps * 16 * D * 4 + 2 * kDecWarps * 16 * 4 +
                      (size_t)kDecMaxEntries * 16 + kDecStages * 8 + 16;
  cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_attn_kernel<D>, dim3(g.n_ctas), dim3(kDecThreads), smem, stream, mk, mv,
                    mq, p);
}

// ---------------------------------------------------------------------------
// Fused decode step, used when every (batch, KV head) unit gets a CTA of its
// own (units <= SMs) and the CNN fits the tensor-core scoring tile: one
// launch per step.  320 threads (the scoring tile's size), per unit:
//   warp 8     cache update: token t-w leaves slot t mod w (to its sink slot,
//              into the retained ring, or dropped), token t takes the slot;
//              the rows are written to global memory, fenced for the async
//              proxy, and the new retained count is published through an
//              mbarrier;
//   warp 9     TMA producer: 64-slot chunks of K and V (one 3-D box each)
//              into a ring of up to 192 KiB.  The window chunks the update cannot touch go first
//              (their copies overlap the update); the chunk holding slot
//              t mod w, the sinks and the retained ring follow once the
//              update has landed;
//   warps 0..NS-1  one per ring stage (NS = 6 at D = 128, 7 at D = 64):
//              chunk c goes to stage and warp c mod NS, so a warp only ever
//              waits for the next phase of its own stage (a phase parity
//              cannot alias).  K Q^T and V^T P^T on m16n8k16 bf16 MMAs with
//              the keys (resp. head dims) as MMA rows and the G query heads as
//              the 8 (or 16) columns, online softmax per chunk, the stage
//              released through an mbarrier -- the warps never wait for one
//              another;
//   warp NS    takes the step ticket (below) once the step index is known,
//              off the path of the copies;
// then the NS (m, l, o) partials are merged in shared memory and o_t,
// lse_t written; when the deferred batch is due the same CTA scores it
// (score_tile_tc, the arithmetic of lte_score).  The step counter lives in
// the cache: every CTA reads meta[0..1], then takes a ticket on meta[3]; the
// last ticket advances t (and n_scored) and resets the ticket.  The partials
// are stored in rows padded to D + 4 floats, so that the lanes of a warp write
// distinct banks.
constexpr int kFuUpdWarp = 8, kFuProdWarp = 9;
constexpr int kFuRingBytes = 192 * 1024;
// ring stages (= attention warps) for head dim D: at most 192 KiB and 7 warps
// (warp NS takes the step ticket)
__host__ __device__ constexpr int fu_stages(int D) {
  return kFuRingBytes / (4 * kDecChunk * D) < 7 ? kFuRingBytes / (4 * kDecChunk * D) : 7;
}

struct FusedParams {
  int Hq, Hkv, G, window, sink, cap, cap_policy, L, score_batch, future;
  float tau, scale_log2;
  const __nv_bfloat16* q_t;
  const __nv_bfloat16* k_t;
  const __nv_bfloat16* v_t;
  __nv_bfloat16* ck;
  __nv_bfloat16* cv;
  int32_t* pos;
  float* win_r;
  int32_t* ret_total;
  int32_t* meta;
  __nv_bfloat16* o_t;
  float* lse_t;
  DevError* err;
  float* ret_r;
};

// The chunks of one step, in issue order: the window chunks except the one
// holding slot t mod w (index kw), then chunk kw, then the sink slots, then
// the retained slots.  nw valid window slots, ns sinks, nr retained (nr is
// known once the update has run).
struct FuChunks {
  int nw, kw, ns, nr, window, sink;
  __device__ __forceinline__ int nwc() const { return (nw + kDecChunk - 1) / kDecChunk; }
  __device__ __forceinline__ int early() const { return nwc() - 1; }
  __device__ __forceinline__ int count() const {
    return nwc() + (ns + kDecChunk - 1) / kDecChunk + (nr + kDecChunk - 1) / kDecChunk;
  }
  __device__ __forceinline__ void get(int c, int& slot0, int& nk) const {
    const int a = nwc();
    if (c < a) {
      const int k = c < a - 1 ? (c < kw ? c : c + 1) : kw;
      slot0 = k * kDecChunk;
      nk = min(kDecChunk, nw - slot0);
      return;
    }
    c -= a;
    const int bs = (ns + kDecChunk - 1) / kDecChunk;
    if (c < bs) {
      slot0 = window + c * kDecChunk;
      nk = min(kDecChunk, ns - c * kDecChunk);
      return;
    }
    c -= bs;
    slot0 = window + sink + c * kDecChunk;
    nk = min(kDecChunk, nr - c * kDecChunk);
  }
};

// bounded wait (1 s) that also gives up when the CTA is aborting
__device__ __forceinline__ bool fu_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                        DevError* err, int where) {
  return mbar_wait_bounded(bar, parity, 1000000000ull, abort_flag, err, where);
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// 8x8 bf16 matrix held one row pair per lane (row lane/4, columns 2(lane%4), +1),
// transposed in registers
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// NT: tiles of 8 query heads per KV head (1 for G <= 8, 2 for G <= 16)
template <int D, int NT>
__global__ void __launch_bounds__(kTcThreads, 1)
decode_fused_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const FusedParams p, const ScoreParams sp, const RingKV<__nv_bfloat16> kv) {
  constexpr int KSTEPS = D / 16, DM = D / 16;
  constexpr int kKV = kDecChunk * D * 2;                  // K or V of one chunk
  constexpr int kStage = 2 * kKV;
  constexpr int NS = fu_stages(D);                        // stages = attention warps
  constexpr int kRowF = D + 4;     // partial rows padded: the per-lane stores hit distinct banks
  extern __shared__ __align__(1024) uint8_t dsm[];
  uint64_t* full = reinterpret_cast<uint64_t*>(dsm + kFuRingBytes);
  uint64_t* empty = full + NS;
  uint64_t* upd = empty + NS;
  int* sh = reinterpret_cast<int*>(upd + 1);   // t, n_scored, retained count, abort, ticket
  volatile int* abort_flag = sh + 3;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = blockIdx.x, b = u / p.Hkv, h = u % p.Hkv;
  if ((smem_u32d(dsm) & 1023u) != 0) {          // swizzle atoms need 1 KiB alignment
    if (tid == 0) record_error(p.err, LTE_ERR_DEVICE, 130);
    return;
  }
  pdl_launch_next();
  if (warp == kFuProdWarp && lane == 0) {         // the descriptors do not depend on the previous step
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_k)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_v)) : "memory");
  }
  if (tid == 0) {
    for (int st = 0; st < NS; ++st) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32d(full + st)));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32d(empty + st)));
    }
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32d(upd)));
    sh[3] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  pdl_wait();              // the previous step has completed: cache and meta are current
  if (tid == 0) {
    sh[0] = p.meta[0];
    sh[1] = p.meta[1];
  }
  __syncthreads();
  if (warp == NS && lane == 0) {
    // the step ticket, taken after the step index was read and used only at the
    // end, so that this round trip is off the path of the copies and the update
    int ticket;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                 : "=r"(ticket)
                 : "l"(p.meta + 3)
                 : "memory");
    sh[4] = ticket;
  }
  const int t = sh[0], n_scored = sh[1];
  const int slot_w = t % p.window, leaving = t - p.window;
  const long long urow = (long long)u * p.L;
  FuChunks ch;
  ch.window = p.window;
  ch.sink = p.sink;
  ch.nw = min(p.window, t + 1);
  ch.kw = slot_w / kDecChunk;
  {
    const int ns = t - p.window + 1;
    ch.ns = ns < 0 ? 0 : (ns > p.sink ? p.sink : ns);
  }
  ch.nr = 0;
  constexpr int kUnknown = 1 << 30;
  // the attention warps' running (m, l, O^T) per head over their chunks
  float o[DM][NT][4];
#pragma unroll
  for (int i = 0; i < DM; ++i)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[i][n][e] = 0.f;
  float m_run[NT][2], l_run[NT][2];
#pragma unroll
  for (int n = 0; n < NT; ++n) m_run[n][0] = m_run[n][1] = -INFINITY, l_run[n][0] = l_run[n][1] = 0.f;

  if (warp == kFuUpdWarp) {
    // ---------------------------------------------------------------- cache update
    constexpr int NV = D * 2 / 16;               // 16-byte vectors per row
    const int e = lane & 15;
    const bool is_v = lane >= 16;
    const long long wrow = (urow + slot_w) * D;
    uint4 new4 = make_uint4(0, 0, 0, 0), old4 = make_uint4(0, 0, 0, 0);
    if (e < NV) {                                // every load before any dependent store
      new4 = reinterpret_cast<const uint4*>((is_v ? p.v_t : p.k_t) + (long long)u * D)[e];
      old4 = reinterpret_cast<const uint4*>((is_v ? p.cv : p.ck) + wrow)[e];
    }
    const int rt = p.ret_total[u];
    int dst = -1, rt_new = rt;
    if (leaving >= 0) {
      const int held = p.pos[urow + slot_w];
      const float r = p.win_r[(long long)u * p.window + slot_w];
      dst = leaving_dst(leaving, held, r, rt, p.window, p.sink, p.cap, p.cap_policy, p.tau,
                        p.pos + urow, p.ret_r + (long long)u * p.cap, p.err, rt_new);
    }
    __syncwarp();                                // every lane has read the slots' positions
    if (e < NV) {
      __nv_bfloat16* base = is_v ? p.cv : p.ck;
      if (dst >= 0) reinterpret_cast<uint4*>(base + (urow + dst) * D)[e] = old4;
      reinterpret_cast<uint4*>(base + wrow)[e] = new4;
    }
    if (lane == 0) {
      if (dst >= 0) p.pos[urow + dst] = leaving;
      if (rt_new != rt) p.ret_total[u] = rt_new;
      p.pos[urow + slot_w] = t;
      p.win_r[(long long)u * p.window + slot_w] = NAN;
      sh[2] = rt_new;
    }
    fence_proxy_async_global();                  // the rows are read next by TMA copies
    __syncwarp();
    if (lane == 0)
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32d(upd)) : "memory");
  } else if (warp == kFuProdWarp) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int n_ch = kUnknown, c = 0;
      const int E = ch.early();
      for (;; ++c) {
        if (c >= E && n_ch == kUnknown) {
          if (!fu_wait(smem_u32d(upd), 0, abort_flag, p.err, 133)) break;
          fence_proxy_async_global();
          ch.nr = min(p.cap, sh[2]);
          n_ch = ch.count();
        }
        if (c >= n_ch) break;
        const int st = c % NS;
        if (c >= NS && !fu_wait(smem_u32d(empty + st), ((c / NS) - 1) & 1, abort_flag, p.err, 134))
          break;
        int slot0, nk;
        ch.get(c, slot0, nk);
        const uint32_t dst = smem_u32d(dsm + st * kStage), bar = smem_u32d(full + st);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(kStage)
                     : "memory");
        const int row = (int)(urow + slot0);
        tma_3d(dst, &tm_k, bar, 0, row, 0);          // all D/64 column halves in one box
        tma_3d(dst + kKV, &tm_v, bar, 0, row, 0);
      }
      // the copies issued last have landed before shared memory is reused
      for (int j = c - NS > 0 ? c - NS : 0; j < c; ++j)
        mbar_wait_d(smem_u32d(full + j % NS), (j / NS) & 1);
    }
  } else if (warp < NS) {
    // ---------------------------------------------------------------- attention
    // Transposed products, keys as the MMA M dimension and the group's query
    // heads as N (NT tiles of 8): S^T = K Q^T (A = K rows by ldmatrix, B = Q^T
    // held in registers) and O^T += V^T P^T (A = V^T by ldmatrix.trans, B =
    // P^T: the S^T accumulator fragment of 16 keys x 8 heads is rounded to
    // bf16 and transposed in registers with movmatrix).
    uint32_t qb[NT][KSTEPS][2];                  // B fragments of Q^T (heads >= G are 0)
    {
      const __nv_bfloat16* q0 = p.q_t + ((long long)b * p.Hq + h * p.G) * D;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int head = n * 8 + (lane >> 2);
#pragma unroll
        for (int kst = 0; kst < KSTEPS; ++kst)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            qb[n][kst][e] = head < p.G ? *reinterpret_cast<const uint32_t*>(
                                             q0 + (long long)head * D + kst * 16 + e * 8 + ((lane & 3) << 1))
                                       : 0u;
      }
    }
    int n_ch = kUnknown;
    const int E = ch.early();
#pragma unroll 1
    for (int c = warp;; c += NS) {
      if (c >= E && n_ch == kUnknown) {
        if (!__all_sync(0xffffffffu, fu_wait(smem_u32d(upd), 0, abort_flag, p.err, 132))) break;
        ch.nr = min(p.cap, sh[2]);
        n_ch = ch.count();
      }
      if (c >= n_ch) break;
      const int st = c % NS;
      if (!__all_sync(0xffffffffu,
                      fu_wait(smem_u32d(full + st), (c / NS) & 1, abort_flag, p.err, 131)))
        break;
      int slot0, nk;
      ch.get(c, slot0, nk);
      const uint8_t* sk = dsm + st * kStage;
      // S^T for the chunk's 64 keys: 4 tiles of 16 keys
      float s[4][NT][4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) s[mt][n][e] = 0.f;
#pragma unroll
      for (int kst = 0; kst < KSTEPS; ++kst)
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          const int r = mt * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
          uint32_t a[4];
          ldsm_x4d(smem_u32d(sk + sw128(kDecChunk, r, kst * 2 + (lane >> 4))), a[0], a[1], a[2],
                   a[3], false);
#pragma unroll
          for (int n = 0; n < NT; ++n) mma_bf16d(s[mt][n], a, qb[n][kst][0], qb[n][kst][1]);
        }
      // per head (columns 2(lane%4), +1 of each n tile): mask, scale, max over the keys
      float mx[NT][2];
#pragma unroll
      for (int n = 0; n < NT; ++n) mx[n][0] = mx[n][1] = -INFINITY;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = mt * 16 + (lane >> 2) + ((e >> 1) << 3);
            s[mt][n][e] = key < nk ? s[mt][n][e] * p.scale_log2 : -INFINITY;
            mx[n][e & 1] = fmaxf(mx[n][e & 1], s[mt][n][e]);
          }
      float corr[NT][2], mu[NT][2];
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float v = mx[n][j];
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
          const float m_new = fmaxf(m_run[n][j], v);
          mu[n][j] = m_new == -INFINITY ? 0.f : m_new;
          corr[n][j] = m_run[n][j] == -INFINITY ? 0.f : exp2f(m_run[n][j] - mu[n][j]);
          m_run[n][j] = m_new;
          l_run[n][j] *= corr[n][j];
        }
#pragma unroll
      for (int i = 0; i < DM; ++i)
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          o[i][n][0] *= corr[n][0]; o[i][n][1] *= corr[n][1];
          o[i][n][2] *= corr[n][0]; o[i][n][3] *= corr[n][1];
        }
      // P^T as B fragments: for key tile mt, {keys 0-7, keys 8-15} x 8 heads
      uint32_t pb[4][NT][2];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          float pv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            pv[e] = exp2f(s[mt][n][e] - mu[n][e & 1]);
            l_run[n][e & 1] += pv[e];
          }
          pb[mt][n][0] = movmatrix_t(pack_bf16d(pv[0], pv[1]));
          pb[mt][n][1] = movmatrix_t(pack_bf16d(pv[2], pv[3]));
        }
      // O^T += V^T P^T: d tiles of 16 x key steps of 16
#pragma unroll
      for (int i = 0; i < DM; ++i)
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          const int r = mt * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int cc = i * 2 + ((lane >> 3) & 1);
          uint32_t a[4];
          ldsm_x4d(smem_u32d(sk + kKV + sw128(kDecChunk, r, cc)), a[0], a[1], a[2], a[3], true);
#pragma unroll
          for (int n = 0; n < NT; ++n) mma_bf16d(o[i][n], a, pb[mt][n][0], pb[mt][n][1]);
        }
      __syncwarp();
      if (lane == 0)
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32d(empty + st))
                     : "memory");
    }
    // finish this warp's per-head sums (lanes with equal lane % 4 share heads)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        l_run[n][j] += __shfl_xor_sync(0xffffffffu, l_run[n][j], 4);
        l_run[n][j] += __shfl_xor_sync(0xffffffffu, l_run[n][j], 8);
        l_run[n][j] += __shfl_xor_sync(0xffffffffu, l_run[n][j], 16);
      }
  }
  __syncthreads();         // every chunk is consumed and every copy has landed
  if (warp < NS) {
    float* o_sh = reinterpret_cast<float*>(dsm);                 // [warps][16 heads][D + 4]
    float* m_sh = o_sh + NS * 16 * kRowF;                        // [warps][16]
    float* l_sh = m_sh + NS * 16;                                // [warps][16]
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int head = n * 8 + ((lane & 3) << 1) + j;
        if (lane < 4) {
          m_sh[warp * 16 + head] = m_run[n][j];
          l_sh[warp * 16 + head] = l_run[n][j];
        }
#pragma unroll
        for (int i = 0; i < DM; ++i) {
          float* row = o_sh + (warp * 16 + head) * kRowF + i * 16 + (lane >> 2);
          row[0] = o[i][n][j];
          row[8] = o[i][n][2 + j];
        }
      }
  }
  __syncthreads();         // the partials are in shared memory
  const bool aborted = *abort_flag != 0;
  if (!aborted) {
    const float* o_sh = reinterpret_cast<const float*>(dsm);
    const float* m_sh = o_sh + NS * 16 * kRowF;
    const float* l_sh = m_sh + NS * 16;
    for (int i2 = tid; i2 < p.G * (D / 4); i2 += kTcThreads) {
      const int g = i2 / (D / 4), d4 = (i2 % (D / 4)) * 4;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NS; ++w) M = fmaxf(M, m_sh[w * 16 + g]);
      float l = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < NS; ++w) {
        const float mw = m_sh[w * 16 + g];
        const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
        l += l_sh[w * 16 + g] * f;
        const float4 ow = *reinterpret_cast<const float4*>(o_sh + (w * 16 + g) * kRowF + d4);
        acc.x += ow.x * f; acc.y += ow.y * f; acc.z += ow.z * f; acc.w += ow.w * f;
      }
      const float inv = 1.f / l;
      __nv_bfloat16* orow = p.o_t + ((long long)b * p.Hq + h * p.G + g) * D + d4;
      *reinterpret_cast<uint2*>(orow) =
          make_uint2(pack_bf16d(acc.x * inv, acc.y * inv), pack_bf16d(acc.z * inv, acc.w * inv));
      if (d4 == 0 && p.lse_t != nullptr)
        p.lse_t[(long long)b * p.Hq + h * p.G + g] = (M + log2f(l)) * 0.69314718055994531f;
    }
  }
  // ---- deferred batched scoring of the oldest scorable tokens of this unit
  const bool due = (t - p.future) - n_scored + 1 >= p.score_batch;
  if (due && !aborted) {
    __syncthreads();       // the partials have been read: shared memory is free
    const int j_end = n_scored + p.score_batch;
    for (int jb = n_scored; jb < j_end; jb += kScoreNT)
      score_tile_tc<RingKV<__nv_bfloat16>>(sp, kv, b, h, jb, j_end, t + 1, dsm);
  }
  // every CTA read meta before taking its ticket: the last one advances the step
  if (tid == 0 && sh[4] == (int)gridDim.x - 1) {
    p.meta[0] = t + 1;
    p.meta[1] = due ? n_scored + p.score_batch : n_scored;
    p.meta[3] = 0;
  }
}

template <int D, int NT>
static cudaError_t launch_fused(const lte_dims* d, const lte_cnn* cnn, const lte_cache* c,
                                const void* q_t, const void* k_t, const void* v_t, void* o_t,
                                float* lse_t, int score_batch, DevError* err, cudaStream_t stream) {
  FusedParams p{};
  p.Hq = d->Hq; p.Hkv = d->Hkv; p.G = d->Hq / d->Hkv; p.window = d->window; p.sink = d->sink;
  p.cap = d->cap; p.cap_policy = d->cap_policy; p.L = d->window + d->sink + d->cap;
  p.score_batch = score_batch;
  p.future = (cnn->k1 - 1 - cnn->past1) + (cnn->k2 - 1 - cnn->past2);
  p.tau = d->tau; p.scale_log2 = d->scale * 1.4426950408889634f;
  p.q_t = (const __nv_bfloat16*)q_t; p.k_t = (const __nv_bfloat16*)k_t;
  p.v_t = (const __nv_bfloat16*)v_t;
  p.ck = (__nv_bfloat16*)c->k; p.cv = (__nv_bfloat16*)c->v; p.pos = c->pos; p.win_r = c->win_r;
  p.ret_total = c->ret_total; p.meta = c->meta; p.ret_r = c->ret_r;
  p.o_t = (__nv_bfloat16*)o_t; p.lse_t = lse_t; p.err = err;
  ScoreParams sp = score_params(d, cnn);
  sp.window = d->window;
  sp.win_r = c->win_r;
  const RingKV<__nv_bfloat16> kv{(const __nv_bfloat16*)c->k, (const __nv_bfloat16*)c->v, d->Hkv,
                                 p.L, d->window, d->D};
  CUtensorMap mk, mv;
  const long long rows = (long long)d->B * d->Hkv * p.L;
  if (!rows_map_halves(&mk, c->k, rows, D, kDecChunk) ||
      !rows_map_halves(&mv, c->v, rows, D, kDecChunk))
    return cudaErrorInvalidValue;
  constexpr int NS = fu_stages(D);
  const size_t smem = kFuRingBytes + (2 * NS + 1) * 8 + 8 * sizeof(int);
  // the merge buffers (8 x 16 x D + 256 floats) and the scoring tile reuse the ring
  cudaError_t e = cudaFuncSetAttribute(decode_fused_kernel<D, NT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_fused_kernel<D, NT>, dim3(d->B * d->Hkv), dim3(kTcThreads), smem, stream, mk,
                    mv, p, sp, kv);
}

cudaError_t decode_step(const lte_dims* d, const lte_cnn* cnn, const lte_cache* c,
                        const void* q_t, const void* k_t, const void* v_t, void* o_t,
                        float* lse_t, int score_batch, DevError* err, void* scratch,
                        cudaStream_t stream) {
  const int n_units = d->B * d->Hkv;
  const int G = d->Hq / d->Hkv;
  float* part = reinterpret_cast<float*>(scratch);
  int32_t* counters = reinterpret_cast<int32_t*>(
      reinterpret_cast<char*>(scratch) +
      (size_t)n_units * dec_geom(d).max_parts * G * (d->D + 4) * sizeof(float));
  // one fused launch when every unit has a CTA of its own and the scorer is the tensor-core tile
  if (dec_geom(d).single && score_tc_supported(cnn->c_hid, cnn->k1, cnn->k2) &&
      score_tc_smem_bytes(d->D, cnn->c_hid, cnn->k2) <= (size_t)kFuRingBytes) {
    const bool g8 = G <= 8;
    if (d->D == 128)
      return g8 ? launch_fused<128, 1>(d, cnn, c, q_t, k_t, v_t, o_t, lse_t, score_batch, err, stream)
                : launch_fused<128, 2>(d, cnn, c, q_t, k_t, v_t, o_t, lse_t, score_batch, err, stream);
    return g8 ? launch_fused<64, 1>(d, cnn, c, q_t, k_t, v_t, o_t, lse_t, score_batch, err, stream)
              : launch_fused<64, 2>(d, cnn, c, q_t, k_t, v_t, o_t, lse_t, score_batch, err, stream);
  }
  cudaError_t e = launch_prep<__nv_bfloat16>(d, cnn, c, k_t, v_t, score_batch, counters, err, stream);
  if (e != cudaSuccess) return e;
  if (d->D == 128) return launch_attn<128>(d, c, q_t, o_t, lse_t, part, counters, err, stream);
  return launch_attn<64>(d, c, q_t, o_t, lse_t, part, counters, err, stream);
}

// ---------------------------------------------------------------------------
// Scratch of lte_decode_step_noalloc, for callers that cannot allocate device
// memory: one file-scope array per device, zero at module load, held until the
// process exits.  Host code must not pass the symbol itself to a kernel (on
// the host it names a stand-in, not device memory): the device address is
// looked up once per device with that device current, and cached.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LTE_NOALLOC_SCRATCH_BYTES];

cudaError_t noalloc_scratch(void** ptr) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  return cudaSuccess;
}

}  // namespace lte
