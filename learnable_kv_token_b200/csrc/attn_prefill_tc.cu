// Prefill sparse attention on 5th-generation tensor cores (tcgen05 + TMEM +
// TMA), bf16 in, fp32 accumulate, head dim 128.
//
// "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention
// and Contextualized Learnable Token Eviction", Fig. 2 caption (right): the
// per-head A-plus-column pattern.  Row t of KV head h attends to
//   S_t = { j < s : j <= t-w } u (t-w, t] u { idx[i] : max(0, n_t-C) <= i < n_t },
//   n_t = cnt[t-w] (0 for t < w).
//
// One CTA computes a 128-row tile: 128/G tokens x the G query heads of one KV
// head (rows token-major), so each K/V tile it loads serves the whole group.
// Keys come in tiles of 64 from up to three ranges: the sink slots and the
// retained slots of the column segment (compacted rows, contiguous) and the
// window band of the key tensor; each tile is one TMA box per 64-column half.
// Warp roles (192 threads):
//   warp 0     TMA producer: Q once, then K and V tiles into a 2-stage ring;
//   warp 1     TMEM owner and MMA issuer (one thread): S = Q K^T into TMEM,
//              O += P V with O resident in TMEM for the whole key loop;
//   warps 2-5  softmax: one thread per row reads its S row from TMEM, applies
//              the attended-set predicate, keeps the running max and sum,
//              writes P (bf16) into a 128B-swizzled shared tile for the PV
//              MMA, and rescales the O row in TMEM only when the running max
//              grew by more than 2^8 (exact: O and l share the reference max);
//              then the epilogue reads O, divides by l and stores bf16.
// The MMA warp issues S_{j+1} before PV_j, so the QK^T of the next tile runs
// while the softmax of this one is computed.  Every mbarrier wait is bounded
// (1 s of global time): on expiry the CTA records LTE_ERR_TIMEOUT in the
// workspace error word, stops issuing work, waits (bounded) for its copies
// and MMAs in flight, frees its TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "lte_common.cuh"
#include "lte_internal.h"

namespace lte {
namespace tc {

constexpr int BM = 128;             // rows per CTA (TMEM lanes)
constexpr int BN = 64;              // keys per tile
constexpr int HD = 128;             // head dim
constexpr int kThreads = 192;
constexpr int kStages = 2;
constexpr uint32_t kQBytes = BM * HD * 2;      // 32 KiB
constexpr uint32_t kQHalf = BM * 128;          // one 64-column half of Q: 16 KiB
constexpr uint32_t kKVBytes = BN * HD * 2;     // 16 KiB (K or V of one tile)
constexpr uint32_t kKVHalf = BN * 128;         // 8 KiB
constexpr uint32_t kPBytes = BM * BN * 2;      // 16 KiB
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKV = kQBytes;                              // stage s: K at +s*32K, V at +16K
constexpr uint32_t kOffP = kOffKV + kStages * 2 * kKVBytes;       // 96 KiB
constexpr uint32_t kOffBar = kOffP + kPBytes;                     // 112 KiB
constexpr uint32_t kSmemBytes = kOffBar + 256;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0, kColO = 64;
constexpr unsigned long long kWaitNs = 1000000000ull;             // bounded waits: 1 s

// barrier slots (8 bytes each) after kOffBar
enum { B_Q = 0, B_KF = 1, B_VF = 3, B_KVE = 5, B_SF = 7, B_SFREE = 8, B_PF = 9, B_PVD = 10,
       B_FIN = 11, kNumBars = 12 };

struct Params {
  int T, Hq, Hkv, G, TOK, sink, window, cap;
  float scale_log2;
  const int32_t* cnt;
  __nv_bfloat16* o;
  Strides4 os;
  float* lse;
  DevError* err;
};

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t sa(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long gtime() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: false if the CTA is aborting or the wait ran out (then aborts).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          DevError* err, int where) {
  if (mbar_try(bar, parity)) return true;
  const unsigned long long t0 = gtime();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (*abort_flag) return false;
    if (gtime() - t0 > kWaitNs) {
      record_error(err, LTE_ERR_TIMEOUT, where);
      *abort_flag = 1;
      return false;
    }
  }
}
// Wait used while shutting down: bounded, ignores the abort flag.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = gtime();
  while (!mbar_try(bar, parity) && gtime() - t0 < kWaitNs) {
  }
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// 128B-swizzled K-major or MN-major shared-memory matrix descriptor (version 1)
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// instruction descriptor, kind::f16: bf16 A/B, fp32 D
__host__ __device__ constexpr uint32_t idesc(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(id), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

#define LTE_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                  "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define LTE_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), \
                  "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])
// 32 consecutive 32-bit TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : LTE_R8(0), LTE_R8(8), LTE_R8(16), LTE_R8(24)
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
          taddr),
      LTE_W8(0), LTE_W8(8), LTE_W8(16), LTE_W8(24)
      : "memory");
}
#undef LTE_R8
#undef LTE_W8
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

struct Tiles {
  int start[3], count[3], ntile[3], total;   // 0: sink slots, 1: retained slots, 2: window band
  __device__ __forceinline__ void at(int it, int& rg, int& key0, int& nk) const {
    rg = 0;
    while (rg < 2 && it >= ntile[rg]) { it -= ntile[rg]; ++rg; }
    key0 = start[rg] + it * BN;
    nk = min(BN, count[rg] - it * BN);
  }
};

__global__ void __launch_bounds__(kThreads, 2)
attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_kc,
                       const __grid_constant__ CUtensorMap tm_vc, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = sa(smem);
  const uint32_t bar0 = sbase + kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffBar + 8 * kNumBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + 8 * kNumBars + 4);

  if ((sbase & 1023u) != 0) {                      // swizzle atoms need 1 KiB alignment
    if (tid == 0) record_error(p.err, LTE_ERR_DEVICE, 110);
    return;
  }
  // ---- tile geometry (identical in every thread)
  const int n_qt = (p.T + p.TOK - 1) / p.TOK;
  const int t0 = (n_qt - 1 - (int)blockIdx.x) * p.TOK;      // heavy (late) tiles first
  const int h = blockIdx.y, b = blockIdx.z, u = b * p.Hkv + h;
  const int t_last = min(t0 + p.TOK - 1, p.T - 1);
  const long long crow = (long long)u * p.T;
  Tiles tl;
  {
    const int n_first = (t0 >= p.window) ? p.cnt[crow + t0 - p.window] : 0;
    const int n_last = (t_last >= p.window) ? p.cnt[crow + t_last - p.window] : 0;
    const int lo_min = n_first - p.cap > 0 ? n_first - p.cap : 0;
    int nsink = t_last - p.window + 1;
    nsink = nsink < 0 ? 0 : (nsink > p.sink ? p.sink : nsink);
    nsink = nsink > p.T ? p.T : nsink;
    int r_start = p.sink + lo_min, r_count = (p.cap > 0 && n_last > lo_min) ? n_last - lo_min : 0;
    if (nsink > 0 && r_count > 0 && r_start - nsink < BN / 2) {   // one slot range [0, end)
      r_count += r_start;
      r_start = 0;
      nsink = 0;
    }
    const int w_lo = t0 - p.window + 1 > 0 ? t0 - p.window + 1 : 0;
    tl.start[0] = 0; tl.count[0] = nsink;
    tl.start[1] = r_start; tl.count[1] = r_count;
    tl.start[2] = w_lo; tl.count[2] = t_last - w_lo + 1;
    tl.total = 0;
    for (int i = 0; i < 3; ++i) { tl.ntile[i] = (tl.count[i] + BN - 1) / BN; tl.total += tl.ntile[i]; }
  }
  const int n_tiles = tl.total;

  if (tid == 0) {
    mbar_init(bar(B_Q), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(B_KF + s), 1);
      mbar_init(bar(B_VF + s), 1);
      mbar_init(bar(B_KVE + s), 1);
    }
    mbar_init(bar(B_SF), 1);
    mbar_init(bar(B_SFREE), 128);
    mbar_init(bar(B_PF), 128);
    mbar_init(bar(B_PVD), 1);
    mbar_init(bar(B_FIN), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     sa(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ======================= TMA producer
    if (lane == 0) {
      int issued = 0;
      mbar_expect_tx(bar(B_Q), kQBytes);
      tma_load_4d(sbase + kOffQ, &tm_q, bar(B_Q), 0, h * p.G, t0, b);
      tma_load_4d(sbase + kOffQ + kQHalf, &tm_q, bar(B_Q), 64, h * p.G, t0, b);
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j & 1, n = j >> 1;
        if (j >= kStages && !mbar_wait(bar(B_KVE + s), (n - 1) & 1, abort_flag, p.err, 104)) break;
        int rg, key0, nk;
        tl.at(j, rg, key0, nk);
        const uint32_t kd = sbase + kOffKV + s * 2 * kKVBytes, vd = kd + kKVBytes;
        mbar_expect_tx(bar(B_KF + s), kKVBytes);
        if (rg == 2) {
          tma_load_4d(kd, &tm_k, bar(B_KF + s), 0, h, key0, b);
          tma_load_4d(kd + kKVHalf, &tm_k, bar(B_KF + s), 64, h, key0, b);
        } else {
          tma_load_3d(kd, &tm_kc, bar(B_KF + s), 0, key0, u);
          tma_load_3d(kd + kKVHalf, &tm_kc, bar(B_KF + s), 64, key0, u);
        }
        mbar_expect_tx(bar(B_VF + s), kKVBytes);
        if (rg == 2) {
          tma_load_4d(vd, &tm_v, bar(B_VF + s), 0, h, key0, b);
          tma_load_4d(vd + kKVHalf, &tm_v, bar(B_VF + s), 64, h, key0, b);
        } else {
          tma_load_3d(vd, &tm_vc, bar(B_VF + s), 0, key0, u);
          tma_load_3d(vd + kKVHalf, &tm_vc, bar(B_VF + s), 64, key0, u);
        }
        issued = j + 1;
      }
      // drain: every issued copy has landed before the CTA may exit
      mbar_drain(bar(B_Q), 0);
      for (int j = issued - kStages > 0 ? issued - kStages : 0; j < issued; ++j) {
        mbar_drain(bar(B_KF + (j & 1)), (j >> 1) & 1);
        mbar_drain(bar(B_VF + (j & 1)), (j >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc(BM, BN, false);
      constexpr uint32_t idO = idesc(BM, HD, true);
      const uint32_t qa = sbase + kOffQ;
      bool ok = mbar_wait(bar(B_Q), 0, abort_flag, p.err, 101);
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j < n_tiles) {
          const int s = j & 1;
          if (j >= 1 && !(ok = mbar_wait(bar(B_SFREE), (j - 1) & 1, abort_flag, p.err, 102))) break;
          if (!(ok = mbar_wait(bar(B_KF + s), (j >> 1) & 1, abort_flag, p.err, 101))) break;
          tc_fence_after();
          const uint32_t kb = sbase + kOffKV + s * 2 * kKVBytes;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint64_t a = sdesc(qa + (kk >> 2) * kQHalf + (kk & 3) * 32, 16, 1024);
            const uint64_t bb = sdesc(kb + (kk >> 2) * kKVHalf + (kk & 3) * 32, 16, 1024);
            mma_f16(tmem + kColS, a, bb, idS, kk > 0);
          }
          mma_commit(bar(B_SF));
        }
        if (j >= 1) {
          const int i = j - 1, s = i & 1;
          if (!(ok = mbar_wait(bar(B_PF), i & 1, abort_flag, p.err, 102))) break;
          if (!(ok = mbar_wait(bar(B_VF + s), (i >> 1) & 1, abort_flag, p.err, 101))) break;
          tc_fence_after();
          const uint32_t vb = sbase + kOffKV + s * 2 * kKVBytes + kKVBytes;
          const uint32_t pa = sbase + kOffP;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t a = sdesc(pa + kk * 32, 16, 1024);
            const uint64_t bb = sdesc(vb + kk * 2048, kKVHalf, 1024);
            mma_f16(tmem + kColO, a, bb, idO, (i > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(B_KVE + s));
          mma_commit(bar(B_PVD));
        }
      }
      // all MMAs issued by this thread are complete before TMEM is released
      mma_commit(bar(B_FIN));
      mbar_drain(bar(B_FIN), 0);
    }
  } else {
    // ======================= softmax + epilogue (warps 2..5, one row per thread)
    const int quad = warp & 3;                     // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const int g = row % p.G, tt = t0 + row / p.G;
    const bool row_ok = tt < p.T;
    int hi_t = 0;
    if (row_ok && tt >= p.window) hi_t = p.cnt[crow + tt - p.window];
    const int lo_t = hi_t - p.cap > 0 ? hi_t - p.cap : 0;
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    uint8_t* prow = smem + kOffP + row * 128;
    for (int j = 0; j < n_tiles; ++j) {
      ok = mbar_wait(bar(B_SF), j & 1, abort_flag, p.err, 103);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;     // tcgen05.ld is warp-collective
      tc_fence_after();
      uint32_t sr[2][32];
      tmem_ld32(lane_addr + kColS, sr[0]);
      tmem_ld32(lane_addr + kColS + 32, sr[1]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(B_SFREE));
      int rg, key0, nk;
      tl.at(j, rg, key0, nk);
      float s[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(sr[c >> 5][c & 31]) * p.scale_log2;
      // attended-set predicate (skipped when the whole tile is inside S_t)
      bool full;
      if (rg == 2) full = nk == BN && key0 > tt - p.window && key0 + BN - 1 <= tt;
      else full = nk == BN && key0 >= p.sink && key0 - p.sink >= lo_t && key0 - p.sink + BN <= hi_t;
      full = full && row_ok;
      if (!full) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int key = key0 + c;
          bool in;
          if (rg == 2) in = key <= tt && key > tt - p.window;
          else if (key < p.sink) in = key <= tt - p.window;
          else in = key - p.sink >= lo_t && key - p.sink < hi_t;
          in = in && c < nk && row_ok;
          if (!in) s[c] = -INFINITY;
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c) mx = fmaxf(mx, s[c]);
      // lazy rescale: move the reference max only when it grew by > 8 (x256)
      const bool need = mx > m_ref + 8.f;
      float corr = 1.f;
      if (need) {
        corr = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - mx);
        m_ref = mx;
        l_sum *= corr;
      }
      const bool any_rescale = __any_sync(0xffffffffu, need && corr != 0.f);
      if (j >= 1) {     // PV_{j-1} done: P buffer free, O up to date
        ok = mbar_wait(bar(B_PVD), (j - 1) & 1, abort_flag, p.err, 103);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        tc_fence_after();
      }
      if (any_rescale) {
#pragma unroll 1
        for (int c0 = 0; c0 < HD; c0 += 32) {
          uint32_t orr[32];
          tmem_ld32(lane_addr + kColO + c0, orr);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * corr);
          tmem_st32(lane_addr + kColO + c0, orr);
        }
        tmem_wait_st();
      }
      const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
      float psum = 0.f;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = exp2f(s[c8 * 8 + 2 * e] - mu);
          const float p1 = exp2f(s[c8 * 8 + 2 * e + 1] - mu);
          psum += p0 + p1;
          __nv_bfloat162 v2 = __floats2bfloat162_rn(p0, p1);
          pk[e] = *reinterpret_cast<uint32_t*>(&v2);
        }
        *reinterpret_cast<uint4*>(prow + ((c8 ^ (row & 7)) << 4)) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      l_sum += psum;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      mbar_arrive(bar(B_PF));
    }
    // ---- epilogue: O / l -> bf16, lse
    if (ok && n_tiles > 0) ok = mbar_wait(bar(B_PVD), (n_tiles - 1) & 1, abort_flag, p.err, 103);
    if (__all_sync(0xffffffffu, ok) && n_tiles > 0) {
      tc_fence_after();
      const float inv = 1.f / l_sum;
      __nv_bfloat16* orow = p.o + (long long)b * p.os.b + (long long)(row_ok ? tt : 0) * p.os.t +
                            (long long)(h * p.G + g) * p.os.h;
#pragma unroll 1
      for (int c0 = 0; c0 < HD; c0 += 32) {
        uint32_t orr[32];
        tmem_ld32(lane_addr + kColO + c0, orr);
        tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 v;
            uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(orr[e + 2 * f]) * inv,
                                                        __uint_as_float(orr[e + 2 * f + 1]) * inv);
              w[f] = *reinterpret_cast<uint32_t*>(&v2);
            }
            *reinterpret_cast<uint4*>(orow + c0 + e) = v;
          }
        }
      }
      if (row_ok && p.lse != nullptr)
        p.lse[((long long)b * p.Hq + h * p.G + g) * p.T + tt] =
            (m_ref + log2f(l_sum)) * 0.69314718055994531f;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

static bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                   const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  auto fn = get_encode();
  if (fn == nullptr) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims,
                  strides_bytes, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace tc

bool attn_prefill_tc_supported(const lte_dims* d) {
  const int G = d->Hq / d->Hkv;
  return d->dtype == LTE_BF16 && d->D == tc::HD && (G == 1 || G == 2 || G == 4 || G == 8 ||
                                                    G == 16);
}

cudaError_t attn_prefill_tc(const PrefillArgs& a, cudaStream_t stream) {
  using namespace tc;
  const lte_dims* d = a.d;
  const int G = d->Hq / d->Hkv, TOK = BM / G;
  CUtensorMap mq, mk, mv, mkc, mvc;
  {
    const cuuint64_t dims[4] = {(cuuint64_t)HD, (cuuint64_t)d->Hq, (cuuint64_t)d->T, (cuuint64_t)d->B};
    const cuuint64_t st[3] = {(cuuint64_t)a.qs.h * 2, (cuuint64_t)a.qs.t * 2, (cuuint64_t)a.qs.b * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)TOK, 1};
    if (!encode(&mq, a.q, 4, dims, st, box)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[4] = {(cuuint64_t)HD, (cuuint64_t)d->Hkv, (cuuint64_t)d->T, (cuuint64_t)d->B};
    const cuuint64_t st[3] = {(cuuint64_t)a.kvs.h * 2, (cuuint64_t)a.kvs.t * 2,
                              (cuuint64_t)a.kvs.b * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)BN, 1};
    if (!encode(&mk, a.k, 4, dims, st, box)) return cudaErrorInvalidValue;
    if (!encode(&mv, a.v, 4, dims, st, box)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t rows = (cuuint64_t)d->sink + d->T;
    const cuuint64_t dims[3] = {(cuuint64_t)HD, rows, (cuuint64_t)d->B * d->Hkv};
    const cuuint64_t st[2] = {(cuuint64_t)HD * 2, rows * HD * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)BN, 1};
    if (!encode(&mkc, a.k_col, 3, dims, st, box)) return cudaErrorInvalidValue;
    if (!encode(&mvc, a.v_col, 3, dims, st, box)) return cudaErrorInvalidValue;
  }
  Params p{};
  p.T = d->T; p.Hq = d->Hq; p.Hkv = d->Hkv; p.G = G; p.TOK = TOK;
  p.sink = d->sink; p.window = d->window; p.cap = d->cap;
  p.scale_log2 = d->scale * 1.4426950408889634f;
  p.cnt = a.cnt;
  p.o = (__nv_bfloat16*)a.o; p.os = a.os; p.lse = a.lse; p.err = a.err;
  cudaError_t e = cudaFuncSetAttribute(attn_prefill_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((d->T + TOK - 1) / TOK, d->Hkv, d->B);
  attn_prefill_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(mq, mk, mv, mkc, mvc, p);
  return cudaGetLastError();
}

}  // namespace lte
