// Retention-score CNN of LTE on 5th-generation tensor cores (tcgen05 + TMEM +
// TMA): bf16 keys and values, fp32 weights, fp32 accumulation.
//
// "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention
// and Contextualized Learnable Token Eviction", Fig. 2 caption: a CNN stack
// over the short-range past and future context of each KV pair yields the
// per-head retention score r_{j,h}.
//
// Layer 1 is one GEMM per tile once its taps are laid out as output columns
// (tap-major, 32 columns per tap, channels c >= c_hid zero):
//   Y[x, kk*32 + c] = sum_ch X[x][ch] * w1[c][ch][kk]            (X = [k; v] rows)
//   u[c][p]         = SiLU(b1[c] + sum_kk Y[p + kk - past1][kk*32 + c])
//   r[j]            = sigmoid(b2 + sum_kk2 sum_c w2[c][kk2] * u[c][j + kk2 - past2])
// with u = 0 at positions outside the tokens.  X is exact in bf16; each fp32
// weight is split into bf16 hi + lo and both products accumulate into the same
// fp32 TMEM accumulator (relative weight error about 2^-17).
//
// Tile: 128 x rows in four blocks of 32 consecutive tokens, block q in TMEM
// lane quadrant q.  Block q holds tokens j0 + q*NW - P + l (l < 32), with
// P = past1 + past2 and NW = 32 - (k1 - 1) - (k2 - 1).  The tap sums and the
// layer-2 sum reach neighbouring rows by warp shuffles, so lane l of block q
// scores token j0 + q*NW + l - P for P <= l < P + NW: the four blocks score
// NT = 4 * NW consecutive tokens (104 for the 5- and 3-tap layers); the rows
// the blocks share are fetched again (from L2).
//
// Persistent pairs of CTAs (a two-CTA cluster on neighbouring SMs), each pair
// bound to one KV head, walk that head's tiles of all sequences, two tiles at
// a time: the leader (cluster rank 0) takes the even tile of a pair-tile, its
// peer the odd one.  Every layer-1 product is one M256 MMA issued by the
// leader for both CTAs (tcgen05 cta_group::2): each CTA supplies its own 128
// x rows as A and holds half of the weight rows (output columns) as B, and
// each CTA's TMEM receives its own rows.  So each SM keeps only half of the
// head's bf16 hi/lo weights resident (converted once), which leaves room for
// an x ring two tiles deep.  Roles per CTA (448 threads):
//   warp 0     TMA producer: one 64-channel chunk of this CTA's tile's x rows
//              (four boxes of 32 rows x 128 B, 128-byte swizzle; rows outside
//              the tokens read as zero) per stage; the bytes of both CTAs'
//              copies of a stage complete on the leader's barrier;
//   warp 1     TMEM owner in both CTAs; in the leader, the MMA issuer (one
//              elected lane): per chunk, four K-steps of 16 channels, each an
//              (hi, lo) pair of M256 x N x K16 MMAs into one of the TMEM
//              accumulators (N = 32 * k1; three of them, N columns apart, when
//              they fit in 512 columns, else two), with every commit signalled
//              to both CTAs;
//   warps 1-13 convert this CTA's half of the head's weights first (warp 0 is
//              already loading);
//   warps 2-5, 6-9, 10-13  the epilogue groups, one per accumulator (pair-
//              tiles i with i mod 3, or mod 2, equal to the group), one lane
//              quadrant per warp (warp w reads quadrant w mod 4): tap sums by
//              shuffles, SiLU, layer 2, sigmoid, r and the mask.  The
//              accumulator goes back to the leader as soon as its columns are
//              in registers.
// Every mbarrier wait is bounded.  A CTA that gives up writes NaN scores
// (mask 0) for the tokens it did not score, so a failure is visible in r.
// The two CTAs meet at a cluster barrier after setting up their barriers and
// TMEM, and again before releasing TMEM and exiting; both reach each after
// bounded work only.
#include <math.h>

#include "lte_common.cuh"
#include "lte_internal.h"
#include "score_cnn.cuh"
#include "tc_ptx.cuh"

namespace lte {
namespace sc5 {

using namespace tc;

constexpr int kThreads = 448;
constexpr int kRows = 128;                 // x rows per tile (TMEM lanes)
constexpr int kBlk = 32;                   // rows per lane quadrant
constexpr uint32_t kChunkB = kRows * 128;  // one 64-channel chunk of a tile: 16 KiB
constexpr uint32_t kBoxB = kBlk * 128;     // one block's rows of a chunk: 4 KiB
constexpr int kMaxStages = 8;
constexpr int kMaxC = 32;                  // hidden channels: one TMEM column per channel and tap
constexpr int kMaxK2 = 9;
constexpr int kMaxAcc = 3;                 // TMEM accumulators (and epilogue groups)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSmemLimit = 227 * 1024;

enum {
  B_FULL = 0, B_EMPTY = kMaxStages, B_YF = 2 * kMaxStages, B_YE = B_YF + kMaxAcc,
  B_FIN = B_YE + kMaxAcc, B_W = B_FIN + 1, kNumBars = B_W + 1
};
constexpr uint32_t kTailFlags = 8 * kNumBars + 8;                      // barriers, abort flag, TMEM slot
constexpr uint32_t kTailW2 = 256;                                     // w2 [k2][32], b1 after the flags
static_assert(kTailFlags <= kTailW2, "barriers and flags fit before the layer-2 weights");
constexpr uint32_t kTailBytes = kTailW2 + kMaxC * (kMaxK2 + 1) * 4;

struct Params {
  int Hkv, D, T_avail, Trow;
  int c_hid, k1, past1, k2, past2;
  int NW, NT, N, n_cc, n_stages;
  int nacc;                                // accumulators in TMEM, N columns apart
  int j_begin, j_end, tiles_per_unit, n_tiles;
  const float *w1, *b1, *w2, *b2;
  int sink;
  float tau;
  float* r;
  uint8_t* mask;
  float* z1;      // non-NULL: write the first layer's pre-activation b1 + W1 * x as
                  // z1[(b * Hkv + h) * c_hid + c][token] (the CNN backward's recompute)
                  // instead of scores
};

__host__ __device__ inline uint32_t w_bytes(int D, int N) { return (uint32_t)(2 * D / 64) * N * 128; }

// NaN scores (mask 0) for the tokens lane `lane` of quadrant q scores in the
// tiles 2u + rank of pair-tiles u = u_from, u_from + step, ... of head h.
__device__ void write_nan_from(const Params& p, int h, int u_from, int step, int rank, int q,
                               int lane) {
  const int P = p.past1 + p.past2;
  if (lane < P || lane >= P + p.NW) return;
  for (int u = u_from; 2 * u + rank < p.n_tiles; u += step) {
    const int t = 2 * u + rank;
    const int b = t / p.tiles_per_unit, j0 = p.j_begin + (t % p.tiles_per_unit) * p.NT;
    const int j = j0 + q * p.NW + lane - P;
    if (j < min(j0 + p.NT, p.j_end)) {
      const long long o = (long long)(b * p.Hkv + h) * p.Trow + j;
      p.r[o] = __int_as_float(0x7fc00000);
      if (p.mask) p.mask[o] = 0;
    }
  }
}

// ---- the CTA pair (two-CTA cluster, tcgen05 cta_group::2)
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The shared::cluster address of this CTA's shared-memory location `a` in CTA `rank`.
__device__ __forceinline__ uint32_t map_rank(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
// Every thread of both CTAs (release / acquire at cluster scope).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// Arrive on a barrier given by its shared::cluster address (either CTA).
__device__ __forceinline__ void arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}
// Bounded, warp-uniform wait (as tc::wwait) on a barrier of this CTA that the
// other CTA's threads arrive on: acquire at cluster scope.
__device__ __forceinline__ bool try_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool wwait_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  bool ok = try_cluster(bar, parity);
  if (!ok) {
    const unsigned long long t0 = gtime();
    while (true) {
      if (try_cluster(bar, parity)) { ok = true; break; }
      if (*abort_flag) break;
      if (gtime() - t0 > kWaitNs) {
        *abort_flag = 1;
        break;
      }
    }
  }
  return __all_sync(0xffffffffu, ok);
}
// Arrive without ordering this thread's memory accesses (the accumulator
// hand-back: the TMEM loads it follows have already completed).
__device__ __forceinline__ void arrive_cluster_relaxed(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}
// A box into this CTA's shared memory whose bytes complete on the leader's
// barrier (`lead_bar`, a shared::cluster address).
__device__ __forceinline__ void tma_load_4d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t lead_bar, int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(lead_bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
// One M256 product of the pair (issued by the leader): A rows 0-127 from the
// leader's shared memory and 128-255 from the peer's, B rows 0..N/2-1 from the
// leader's and N/2..N-1 from the peer's, both at the descriptors' offsets; D
// rows go to the TMEM of the CTA that supplied them.
__device__ __forceinline__ void mma2_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(id), "r"(accumulate)
      : "memory");
}
// One arrival on barrier `bar` (same offset) in both CTAs once this thread's
// earlier MMAs have completed.
__device__ __forceinline__ void mma2_commit_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}

// This CTA's half of the head's w1 as bf16 hi + lo: weight rows (output
// columns) n = kk*32 + c with n0 <= n < n0 + N/2, K-major with 128-byte
// swizzle: chunk cc of 64 input channels holds local rows m = n - n0 of 128
// bytes, and 16-byte group k8 of row m sits at ((k8 ^ (m & 7)) << 4).  One
// unit = (channel c, group of 8 input channels): its 8 x K1 weights are
// contiguous in w1 (16-byte aligned), read as 2*K1 float4 loads, and give one
// 16-byte hi store and one lo store per tap whose row is this CTA's.
// Threads me = 0 .. kThreads-33 share the units, kA units in flight per thread.
template <int K1>
__device__ __forceinline__ void convert_w(const Params& p, int h, uint8_t* smem, uint32_t wb, int me,
                                          int n0) {
  constexpr int nt = kThreads - 32, kA = K1 <= 5 ? 2 : 1;
  const int twoD = 2 * p.D, G8 = twoD / 8, n_units = kMaxC * G8;
  const float* w1h = p.w1 + (long long)h * p.c_hid * twoD * K1;
  for (int u0 = me; u0 < n_units; u0 += kA * nt) {
    float4 x[kA][2 * K1];
#pragma unroll
    for (int a = 0; a < kA; ++a) {
      const int u = u0 + a * nt, c = u / G8, gi = u % G8;
      const bool live = u < n_units && c < p.c_hid;
      const float4* src = reinterpret_cast<const float4*>(w1h + ((long long)c * twoD + gi * 8) * K1);
#pragma unroll
      for (int e = 0; e < 2 * K1; ++e) x[a][e] = live ? __ldg(src + e) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int a = 0; a < kA; ++a) {
      const int u = u0 + a * nt, c = u / G8, gi = u % G8;
      if (u >= n_units) break;
      const float* f = reinterpret_cast<const float*>(x[a]);   // f[e*K1 + kk]: channel 8gi+e, tap kk
#pragma unroll
      for (int kk = 0; kk < K1; ++kk) {
        const int m = kk * 32 + c - n0, cc = gi >> 3, k8 = gi & 7;
        if (m < 0 || m >= p.N / 2) continue;
        const uint32_t off = (uint32_t)cc * (p.N / 2) * 128 + m * 128 + ((k8 ^ (m & 7)) << 4);
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float w0 = f[(2 * e) * K1 + kk], w1 = f[(2 * e + 1) * K1 + kk];
          const __nv_bfloat16 h0 = __float2bfloat16_rn(w0), h1 = __float2bfloat16_rn(w1);
          const __nv_bfloat16 l0 = __float2bfloat16_rn(w0 - __bfloat162float(h0));
          const __nv_bfloat16 l1 = __float2bfloat16_rn(w1 - __bfloat162float(h1));
          hw[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
          lw[e] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
        }
        *reinterpret_cast<uint4*>(smem + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(smem + wb + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
    }
  }
}

// Wait for this thread's TMEM loads, with `r` (the destination of the last
// one) tied to the wait so that no read of it is scheduled before the wait.
__device__ __forceinline__ void wait_ld_into(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                 "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]),
                 "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
                 "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]),
                 "+r"(r[31])
               :
               : "memory");
}

// SiLU of the hidden layer: x / (1 + e^-x) with the fast exponential and the
// fast division intrinsic (relative error a few ulp; a denominator above 2^126,
// x below about -87, gives 0 or -0, against a true value under 1e-36).  The
// IEEE reciprocal it replaces branches to a slow path that kept the 32
// channels of a row from overlapping.
__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.f + __expf(-x)); }

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
score_tcgen05_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = sa(smem);
  const uint32_t wb = w_bytes(p.D, p.N / 2);          // this CTA's weight rows, hi (lo after them)
  const uint32_t off_ring = 2 * wb, off_tail = off_ring + p.n_stages * kChunkB;
  uint8_t* tail = smem + off_tail;
  const uint32_t bar0 = sbase + off_tail;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tail + 8 * kNumBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tail + 8 * kNumBars + 4);
  float* w2s = reinterpret_cast<float*>(tail + kTailW2);      // [k2][32], zero past c_hid
  float* b1s = w2s + kMaxC * p.k2;                            // [32]

  const int rank = (int)cluster_rank();               // 0: the leader, which issues the MMAs
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int h = pair % p.Hkv;
  const int slot = pair / p.Hkv, n_slots = n_pairs / p.Hkv;
  const int n_pt = (p.n_tiles + 1) >> 1;              // pair-tiles of a head
  const int P = p.past1 + p.past2;

  if ((sbase & 1023u) != 0) {                    // swizzle atoms need 1 KiB alignment (same in both CTAs)
    if (warp >= 2 && warp < 6 && p.z1 == nullptr)
      write_nan_from(p, h, slot, n_slots, rank, warp & 3, lane);
    return;
  }
  if (tid == 0) {
    for (int s = 0; s < p.n_stages; ++s) {
      mbar_init(bar(B_FULL + s), 1);             // the leader's: its arrival, both CTAs' bytes
      mbar_init(bar(B_EMPTY + s), 1);
    }
    for (int x = 0; x < kMaxAcc; ++x) {
      mbar_init(bar(B_YF + x), 1);
      mbar_init(bar(B_YE + x), 8);               // the leader's: one elected lane per epilogue warp of both CTAs
    }
    mbar_init(bar(B_FIN), 1);
    mbar_init(bar(B_W), 2);                      // the leader's: one arrival per CTA, weights in place
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {                               // the same warp in both CTAs allocates for the pair
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     sa(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  for (int i = tid; i < kMaxC * p.k2; i += kThreads) {
    const int kk = i / kMaxC, c = i % kMaxC;
    w2s[i] = c < p.c_hid ? p.w2[((long long)h * p.c_hid + c) * p.k2 + kk] : 0.f;
  }
  for (int c = tid; c < kMaxC; c += kThreads) b1s[c] = c < p.c_hid ? p.b1[h * p.c_hid + c] : 0.f;
  tc_fence_before();
  __syncthreads();
  cluster_sync();                                // both CTAs' barriers exist before any crosses over
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================================================================ TMA producer
    int g = 0;
    bool ok = true;
    const int cc_k = p.D / 64;
    for (int u = slot; ok && u < n_pt; u += n_slots) {
      // the peer of an odd head's last pair-tile reloads the leader's tile and discards its rows
      const int t = min(2 * u + rank, p.n_tiles - 1);
      const int b = t / p.tiles_per_unit, j0 = p.j_begin + (t % p.tiles_per_unit) * p.NT;
      for (int cc = 0; cc < p.n_cc; ++cc, ++g) {
        const int st = g % p.n_stages, use = g / p.n_stages;
        if (use >= 1 && !(ok = wwait(bar(B_EMPTY + st), (use - 1) & 1, abort_flag, nullptr, 0)))
          break;
        if (elect_one()) {
          const uint32_t dst = sbase + off_ring + st * kChunkB;
          const uint32_t lead_full = map_rank(bar(B_FULL + st), 0);
          const CUtensorMap* map = cc < cc_k ? &tm_k : &tm_v;
          const int c0 = (cc % cc_k) * 64;
          if (rank == 0) mbar_expect_tx(bar(B_FULL + st), 2 * kChunkB);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            tma_load_4d_pair(dst + q * kBoxB, map, lead_full, c0, h, j0 + q * p.NW - P, b);
        }
        __syncwarp();
      }
    }
    // every issued copy (of both CTAs) has landed before the pair may exit: the
    // leader's full barriers count both CTAs' bytes, and the peer stays until
    // the closing cluster barrier
    if (rank == 0)
      for (int q = g - p.n_stages > 0 ? g - p.n_stages : 0; q < g; ++q)
        mbar_drain(bar(B_FULL + q % p.n_stages), (q / p.n_stages) & 1);
  } else {
    // ================================================================ weights
    const int n0 = rank * (p.N / 2);
    switch (p.k1) {
      case 1: convert_w<1>(p, h, smem, wb, tid - 32, n0); break;
      case 2: convert_w<2>(p, h, smem, wb, tid - 32, n0); break;
      case 3: convert_w<3>(p, h, smem, wb, tid - 32, n0); break;
      case 4: convert_w<4>(p, h, smem, wb, tid - 32, n0); break;
      case 5: convert_w<5>(p, h, smem, wb, tid - 32, n0); break;
      case 6: convert_w<6>(p, h, smem, wb, tid - 32, n0); break;
      case 7: convert_w<7>(p, h, smem, wb, tid - 32, n0); break;
      default: convert_w<8>(p, h, smem, wb, tid - 32, n0); break;
    }
    fence_proxy_async();                            // generic writes -> tensor-core reads
    asm volatile("bar.sync 1, %0;" ::"n"(kThreads - 32) : "memory");
    if (tid == 32) arrive_cluster(map_rank(bar(B_W), 0));   // this CTA's weight half is in place

    if (warp == 1) {
      if (rank == 0) {
        // ========================================================== MMA issuer (leader)
        const uint32_t idy = idesc(2 * kRows, p.N, false);
        const uint64_t da0 = sdesc(sbase + off_ring, 16, 1024);
        const uint64_t dh0 = sdesc(sbase, 16, 1024);
        const uint64_t dl0 = sdesc(sbase + wb, 16, 1024);
        int g = 0, i = 0;
        bool ok = wwait_cluster(bar(B_W), 0, abort_flag);
        for (int u = slot; ok && u < n_pt; u += n_slots, ++i) {
          const int yb = i % p.nacc;
          if (i >= p.nacc &&
              !(ok = wwait_cluster(bar(B_YE + yb), ((i / p.nacc) - 1) & 1, abort_flag)))
            break;
          tc_fence_after();
          const uint32_t dy = tmem + (uint32_t)(yb * p.N);
          for (int cc = 0; cc < p.n_cc; ++cc, ++g) {
            const int st = g % p.n_stages;
            if (!(ok = wwait(bar(B_FULL + st), (g / p.n_stages) & 1, abort_flag, nullptr, 0))) break;
            tc_fence_after();
            if (elect_one()) {
              const uint64_t da = da0 + ((st * kChunkB) >> 4);
              const uint64_t dwo = (uint64_t)((cc * (p.N / 2) * 128) >> 4);
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                mma2_f16(dy, da + 2 * ks, dh0 + dwo + 2 * ks, idy, (cc | ks) != 0 ? 1u : 0u);
                mma2_f16(dy, da + 2 * ks, dl0 + dwo + 2 * ks, idy, 1u);
              }
              mma2_commit_both(bar(B_EMPTY + st));    // the stage frees in both CTAs once these ran
            }
            __syncwarp();
          }
          if (!ok) break;
          if (elect_one()) mma2_commit_both(bar(B_YF + yb));
          __syncwarp();
        }
        if (elect_one()) mma2_commit_both(bar(B_FIN));  // every MMA of the pair has completed
        __syncwarp();
        mbar_drain(bar(B_FIN), 0);
      }
    } else if (warp >= 2 && (warp - 2) >> 2 < p.nacc) {
      // ============================================================ epilogue
      // group eg (warps 2-5, 6-9 or 10-13) takes the pair-tiles of accumulator
      // eg; warp w reads TMEM lane quadrant w % 4
      const int q = warp & 3, eg = (warp - 2) >> 2;
      const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(eg * p.N);
      const uint32_t ye_lead = map_rank(bar(B_YE + eg), 0);
      int i = eg, u = slot + eg * n_slots;
      bool ok = true;
      for (; u < n_pt; u += p.nacc * n_slots, i += p.nacc) {
        if (!(ok = wwait(bar(B_YF + eg), (i / p.nacc) & 1, abort_flag, nullptr, 0))) break;
        tc_fence_after();
        const int t = 2 * u + rank;
        const bool live = t < p.n_tiles;               // this CTA's rows belong to a tile
        const int tt = live ? t : p.n_tiles - 1;
        const int b = tt / p.tiles_per_unit, j0 = p.j_begin + (tt % p.tiles_per_unit) * p.NT;
        const int tok = j0 + q * p.NW - P + lane;       // token of this lane's row
        float z[kMaxC];
#pragma unroll
        for (int c = 0; c < kMaxC; ++c) z[c] = 0.f;
        // taps in order; the next tap's columns load while this one's are summed
        uint32_t y0[32], y1[32];
        tmem_ld32(lane_addr, y0);
        wait_ld_into(y0);
        for (int kk = 0; kk < p.k1; kk += 2) {
          const bool has1 = kk + 1 < p.k1, has2 = kk + 2 < p.k1;
          if (has1) tmem_ld32(lane_addr + (kk + 1) * 32, y1);
          const int src0 = lane + kk - p.past1;         // row p + kk - past1 of this tap
#pragma unroll
          for (int c = 0; c < kMaxC; ++c) z[c] += __shfl_sync(0xffffffffu, __uint_as_float(y0[c]), src0);
          if (has1) {
            wait_ld_into(y1);
            if (has2) tmem_ld32(lane_addr + (kk + 2) * 32, y0);
            const int src1 = src0 + 1;
#pragma unroll
            for (int c = 0; c < kMaxC; ++c) z[c] += __shfl_sync(0xffffffffu, __uint_as_float(y1[c]), src1);
            if (has2) wait_ld_into(y0);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_cluster_relaxed(ye_lead); // the accumulator may be overwritten
        if (!live) continue;
        if (p.z1 != nullptr) {                          // the pre-activation, this lane's token
          if (lane >= P && lane < P + p.NW && tok < min(j0 + p.NT, p.j_end)) {
            float* zo = p.z1 + (long long)(b * p.Hkv + h) * p.c_hid * p.Trow + tok;
#pragma unroll
            for (int c = 0; c < kMaxC; ++c)
              if (c < p.c_hid) zo[(long long)c * p.Trow] = b1s[c] + z[c];
          }
          continue;
        }
        const bool in_seq = tok >= 0 && tok < p.T_avail;
#pragma unroll
        for (int c = 0; c < kMaxC; c += 4) {
          const float4 bb = *reinterpret_cast<const float4*>(b1s + c);
          z[c] = in_seq ? silu_fast(bb.x + z[c]) : 0.f;
          z[c + 1] = in_seq ? silu_fast(bb.y + z[c + 1]) : 0.f;
          z[c + 2] = in_seq ? silu_fast(bb.z + z[c + 2]) : 0.f;
          z[c + 3] = in_seq ? silu_fast(bb.w + z[c + 3]) : 0.f;
        }
        float acc = 0.f;
        for (int kk = 0; kk < p.k2; ++kk) {             // layer 2, taps in order
          const float* wk = w2s + kk * kMaxC;
          float part = 0.f;
#pragma unroll
          for (int c = 0; c < kMaxC; c += 4) {
            const float4 w = *reinterpret_cast<const float4*>(wk + c);
            part = fmaf(w.x, z[c], part);
            part = fmaf(w.y, z[c + 1], part);
            part = fmaf(w.z, z[c + 2], part);
            part = fmaf(w.w, z[c + 3], part);
          }
          acc += __shfl_sync(0xffffffffu, part, lane + kk - p.past2);
        }
        if (lane >= P && lane < P + p.NW && tok < min(j0 + p.NT, p.j_end)) {
          const float r = sigmoidf_(p.b2[h] + acc);
          const long long o = (long long)(b * p.Hkv + h) * p.Trow + tok;
          p.r[o] = r;
          if (p.mask) p.mask[o] = (tok >= p.sink && r >= p.tau) ? 1 : 0;
        }
      }
      if (!ok && p.z1 == nullptr) write_nan_from(p, h, u, p.nacc * n_slots, rank, q, lane);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();            // neither CTA leaves while the other may still reach its memory
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// stages of the x ring that fit beside a CTA's half of the weights (0 if the
// shape does not fit)
static int ring_stages(int D, int N) {
  const long long room = (long long)kSmemLimit - 2ll * w_bytes(D, N / 2) - kTailBytes;
  const long long st = room / kChunkB;
  return st < 2 ? 0 : (st > kMaxStages ? kMaxStages : (int)st);
}

}  // namespace sc5

bool score_tcgen05_supported(const lte_dims* d, const lte_cnn* cnn, Strides4 s) {
  using namespace sc5;
  if (d->dtype != LTE_BF16 || (d->D != 64 && d->D != 128)) return false;
  if (cnn->c_hid < 1 || cnn->c_hid > kMaxC || cnn->k1 < 1 || 32 * cnn->k1 > 256 ||
      cnn->k2 < 1 || cnn->k2 > kMaxK2)
    return false;
  if (32 - (cnn->k1 - 1) - (cnn->k2 - 1) < 8) return false;      // scored lanes per block
  if (s.h % 8 != 0 || s.t % 8 != 0 || s.b % 8 != 0) return false; // 16-byte TMA strides
  if ((reinterpret_cast<uintptr_t>(cnn->w1) & 15) != 0) return false;  // float4 weight loads
  return ring_stages(d->D, 32 * cnn->k1) >= 2;
}

cudaError_t score_tcgen05(const lte_dims* d, const lte_cnn* cnn, const void* k, const void* v,
                          Strides4 s, int j_begin, int j_end, float* r, uint8_t* mask,
                          cudaStream_t stream, float* z1) {
  using namespace sc5;
  Params p{};
  p.Hkv = d->Hkv; p.D = d->D; p.T_avail = d->T; p.Trow = d->T;
  p.c_hid = cnn->c_hid; p.k1 = cnn->k1; p.past1 = cnn->past1; p.k2 = cnn->k2; p.past2 = cnn->past2;
  p.NW = 32 - (p.k1 - 1) - (p.k2 - 1);
  p.NT = 4 * p.NW;
  p.N = 32 * p.k1;
  p.n_cc = 2 * d->D / 64;
  p.n_stages = ring_stages(d->D, p.N);
  p.nacc = 512 / p.N < kMaxAcc ? 512 / p.N : kMaxAcc;
  p.j_begin = j_begin; p.j_end = j_end;
  p.tiles_per_unit = (j_end - j_begin + p.NT - 1) / p.NT;
  p.n_tiles = d->B * p.tiles_per_unit;
  p.w1 = cnn->w1; p.b1 = cnn->b1; p.w2 = cnn->w2; p.b2 = cnn->b2;
  p.sink = d->sink; p.tau = d->tau; p.r = r; p.mask = mask; p.z1 = z1;
  if (p.n_tiles == 0) return cudaSuccess;
  CUtensorMap mk, mv;
  {
    const cuuint64_t dims[4] = {(cuuint64_t)d->D, (cuuint64_t)d->Hkv, (cuuint64_t)d->T,
                                (cuuint64_t)d->B};
    const cuuint64_t st[3] = {(cuuint64_t)s.h * 2, (cuuint64_t)s.t * 2, (cuuint64_t)s.b * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)kBlk, 1};
    if (!tc::encode(&mk, k, 4, dims, st, box)) return cudaErrorInvalidValue;
    if (!tc::encode(&mv, v, 4, dims, st, box)) return cudaErrorInvalidValue;
  }
  const uint32_t smem = 2 * w_bytes(d->D, p.N / 2) + p.n_stages * kChunkB + kTailBytes;
  cudaError_t e = cudaFuncSetAttribute(score_tcgen05_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // CTA pairs resident at once (one CTA per SM; a GPC with an odd number of
  // SMs leaves one out), cached per device and shared-memory size
  static int cached_dev[8] = {-1, -1, -1, -1, -1, -1, -1, -1};
  static uint32_t cached_smem[8];
  static int cached_pairs[8];
  int dev = 0, n_sm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  const int ci = dev & 7;
  int pairs = 0;
  if (cached_dev[ci] == dev && cached_smem[ci] == smem) {
    pairs = cached_pairs[ci];
  } else {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * (unsigned)(n_sm / 2), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    if (cudaOccupancyMaxActiveClusters(&pairs, score_tcgen05_kernel, &cfg) != cudaSuccess ||
        pairs < 1) {
      (void)cudaGetLastError();
      pairs = n_sm / 2;
    }
    cached_pairs[ci] = pairs;
    cached_smem[ci] = smem;
    cached_dev[ci] = dev;
  }
  long long slots = pairs / d->Hkv;              // pairs per KV head
  if (slots < 1) slots = 1;
  const int n_pt = (p.n_tiles + 1) / 2;
  if (slots > n_pt) slots = n_pt;
  score_tcgen05_kernel<<<(unsigned)(2 * slots * d->Hkv), kThreads, smem, stream>>>(mk, mv, p);
  return cudaGetLastError();
}

}  // namespace lte
