// Gated linear attention prefill on 5th-generation tensor cores (tcgen05 +
// TMEM), bf16 q/k/v/o, fp32 gates, fp32 state.
//
// "Sparse Linear Attention: Viewing SWA from the Perspective of Linear
// Attention", section "Background: Linear attention": S_t = S_{t-1} A_t +
// v_t k_t^T, o_t = S_t q_t, here with A_t = diag(a_t).  The chunk-wise form
// (L = 64 tokens, m = 31 the chunk middle, b_t = sum_{i<=t} log a_i within the
// chunk, x_t = e^{b_t - b_m} per key channel):
//   Q~_t = q_t x_t,  K~_s = k_s / x_s,  Khat_s = k_s e^{b_last - b_s} = K~_s e^{b_last - b_m}
//   A    = tril(Q~ K~^T)                                   (64 x 64)
//   O    = A V + Q~ (S_0 diag(e^{b_m}))^T                  (64 x 128)
//   S_L  = S_0 diag(e^{b_last}) + V^T Khat                 (128 x 128)
// The factors are running products of the gates (of a within the second half,
// of 1/a backwards through the first), so no logarithm or exponential is
// evaluated.
//
// One CTA (512 threads) per (batch, head) walks the chunks in order, in two
// warp groups that work on consecutive chunks at once:
//   gate group (warps 8-15), chunk c + 1: waits for its inputs (q, k, v in
//     128-byte-swizzled halves and the gates, seven TMA copies into one of two
//     shared input sets); thread (j, half) walks key channel j through half of
//     the chunk (factors x_t over the gates, in place); a 16-byte pass writes
//     Q~ and K~ in place and Khat into the set's own buffer; then it signals
//     the TMEM group;
//   TMEM group (warps 0-7; warp w owns TMEM lanes 32 (w % 4) .. + 31 and, in
//     passes over TMEM, one half of the columns), chunk c: A = Q~ K~^T
//     (M = 64) runs while a pass over the state turns S_0 into its bf16 copy
//     S_0 diag(e^{b_m}) (the B operand of O) and into S_0 diag(e^{b_last});
//     the masked A goes to shared memory as bf16 (over the set's consumed gate
//     table), then O = A V + Q~ S_0'^T (M = 64, K = 64 + 128) and
//     S += V^T Khat (M = 128, K = 64) run; one thread requests chunk c + 2's
//     inputs into the freed set, and O is staged as bf16 in the S_0' buffer
//     and written by TMA stores.
// TMEM holds the fp32 state S (columns 0-127, lane = value channel) for the
// whole sequence and one 64-row accumulator (columns 128-255: A of a chunk,
// then its O; a 64-row accumulator keeps row r in lane 32 (r / 16) + r % 16).
// Range.  The factors x_t and 1/x_t are products of up to 32 gates (or their
// reciprocals), so the chunk form needs them inside the fp32/bf16 exponent
// range.  The gate group checks every chunk: when some key channel's product
// of 32 gates falls below 2^-100 (a gate near 0 -- or exactly 0 -- within a
// chunk), that chunk instead runs the recurrence itself, token by token, in
// fp32 on the state held in registers (the TMEM group: thread (row, half)
// updates S[row, 64 half .. + 63], reading the raw gates from global memory,
// and the halves' partial o_t[row] are added through shared memory).  So every gate in [0, 1] gives the recurrence's
// result; only the speed of such chunks differs.
// Every mbarrier wait is bounded; a CTA that gives up writes NaN into its
// final state, so the failure is visible to the caller.
#include <math.h>

#include "lte_common.cuh"
#include "lte_internal.h"
#include "tc_ptx.cuh"

namespace lte {
namespace glatc {

using namespace tc;

constexpr int L = 64, DK = 128, DV = 128;
constexpr int kThreads = 512;
constexpr int kGroup = 256;                        // threads per warp group
constexpr uint32_t kTile = L * 256;                 // [64 rows][128] bf16 as two 64-column halves
constexpr uint32_t kHalf = L * 128;                 // one 64-column half of such a tile
constexpr uint32_t kSetQ = 0, kSetK = kTile, kSetV = 2 * kTile, kSetA = 3 * kTile;
// an input set: q, k, v tiles, the gates [64][128] fp32 (then the decay
// factors, then the masked A [64][64] bf16 in one 128B-swizzled half) and
// Khat [64][128] bf16
constexpr uint32_t kSetKhat = 3 * kTile + L * DK * 4;
constexpr uint32_t kSet = kSetKhat + kTile;
constexpr uint32_t kSb = 2 * kSet;                  // S_0 diag(e^{b_m}) [128][128] bf16 (two halves)
constexpr uint32_t kLam = kSb + DV * 256;           // per set: e^{b_m}, e^{b_last - b_m} per key channel
constexpr uint32_t kBar = kLam + 2 * 2 * DK * 4;    // mbarriers: MMA, inputs landed x2, gates done x2
constexpr uint32_t kSmem = kBar + 64;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0, kColAO = 128;
constexpr unsigned long long kWait = 1000000000ull;
static_assert(kSmem <= 227 * 1024, "shared memory");

// byte offset of 16-byte chunk c16 (0..15 over 128 columns) of row r in a
// [rows][128] bf16 tile stored as two 128B-swizzled 64-column halves
__device__ __forceinline__ uint32_t swz(int rows, int r, int c16) {
  return (uint32_t)((c16 >> 3) * rows * 128 + r * 128 + (((c16 & 7) ^ (r & 7)) << 4));
}
__device__ __forceinline__ float rcp_approx(float x) {   // within 1 ulp
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// instruction descriptor, kind::f16: bf16 A/B, fp32 D; a_mn / b_mn: the operand
// is stored M- (resp. N-) contiguous instead of K-contiguous
__device__ __forceinline__ uint32_t idesc2(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// AND of `v` over the `n` threads of named barrier `id` (all of them call it)
__device__ __forceinline__ bool group_and(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, %2, %3, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void group_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
constexpr int kBarGate = 1, kBarTmem = 2;                // named barriers of the two warp groups

__global__ void __launch_bounds__(kThreads, 1)
gla_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
                      const __grid_constant__ CUtensorMap tm_o, int T, int H,
                      const float* __restrict__ a_raw, float* __restrict__ state) {
  extern __shared__ __align__(1024) uint8_t sm[];
  const int bh = blockIdx.x, b = bh / H, hd = bh % H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t s0 = sa(sm);
  const uint32_t bar_mma = s0 + kBar;                    // MMA completion (TMEM group)
  const uint32_t bar_in = s0 + kBar + 8;                 // inputs of set s landed: + 8 s
  const uint32_t bar_g = s0 + kBar + 24;                 // gate work of set s done: + 8 s
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kBar + 40);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kBar + 44);
  volatile int* exact = reinterpret_cast<volatile int*>(sm + kBar + 48);   // per set: 1 = recurrence
  float* st = state + (long long)bh * DV * DK;
  const int n_chunks = T / L;

  if ((s0 & 1023u) != 0) {                               // swizzle atoms need 1 KiB alignment
    for (int i = tid; i < DV * DK; i += kThreads) st[i] = __int_as_float(0x7fc00000);
    return;
  }
  if (tid == 0) {
    mbar_init(bar_mma, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_in + 8 * s, 1);
      mbar_init(bar_g + 8 * s, 1);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
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

  // inputs of chunk c -> input set c mod 2 (seven TMA copies, issued by the caller)
  auto load_chunk = [&](int c) {
    const int set = c & 1;
    const uint32_t sb = s0 + set * kSet, fb = bar_in + 8 * set;
    mbar_expect_tx(fb, 3 * kTile + L * DK * 4);
    for (int h2 = 0; h2 < 2; ++h2) {
      tma_load_4d(sb + kSetQ + h2 * kHalf, &tm_q, fb, h2 * 64, hd, c * L, b);
      tma_load_4d(sb + kSetK + h2 * kHalf, &tm_k, fb, h2 * 64, hd, c * L, b);
      tma_load_4d(sb + kSetV + h2 * kHalf, &tm_v, fb, h2 * 64, hd, c * L, b);
    }
    tma_load_4d(sb + kSetA, &tm_a, fb, 0, hd, c * L, b);
  };
  int n_issued = n_chunks < 2 ? n_chunks : 2;            // meaningful in thread 0
  if (tid == 0)
    for (int c = 0; c < n_issued; ++c) load_chunk(c);
  bool ok = true;

  if (tid >= kGroup) {
    // ================================================================ gate group
    const int gt = tid - kGroup;
    for (int c = 0; c < n_chunks; ++c) {
      const int set = c & 1;
      uint8_t* sset = sm + set * kSet;
      float* lam_m = reinterpret_cast<float*>(sm + kLam + set * 2 * DK * 4);
      float* lam_r = lam_m + DK;
      ok = mbar_wait_bounded(bar_in + 8 * set, (c >> 1) & 1, kWait, abort_flag, nullptr, 0);
      if (!(ok = group_and(kBarGate, kGroup, ok))) break;
      // ---- decay factors x_t over the gates (in place): thread (j, half) walks
      // key channel j backwards through the first half (product of 1/a over
      // t < i <= m) or forwards through the second (product of a over m < i <= t)
      // The chunk form is used only when, in every channel, the product of each
      // half's 32 gates is >= 2^-100 (then every factor and its reciprocal stays
      // within 2^+-100); otherwise the table keeps the raw gates for the
      // recurrence (`exact`).  NaN or zero gates fail the test too.
      bool in_range;
      {
        const int j = gt & (DK - 1), half = gt >> 7;
        float* Xj = reinterpret_cast<float*>(sset + kSetA) + half * 32 * DK + j;
        float g[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) g[i] = Xj[i * DK];
        float pa = 1.f;
        if (half == 0) {
          float pr = 1.f;
#pragma unroll
          for (int i = 31; i >= 0; --i) {
            const float ai = g[i];
            g[i] = pr;
            pr *= rcp_approx(ai);
            pa *= ai;
          }
          in_range = pa >= 0x1p-100f && pr <= 0x1p100f;
          lam_m[j] = pa;                                   // e^{b_m}
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            pa *= g[i];
            g[i] = pa;
          }
          in_range = pa >= 0x1p-100f;
          lam_r[j] = pa;                                   // e^{b_last - b_m}
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) Xj[i * DK] = g[i];
      }
      // one barrier both publishes the factors and takes the vote (the exact
      // path reads the raw gates from global memory)
      in_range = group_and(kBarGate, kGroup, in_range);
      if (!in_range) {                                     // chunk c runs the recurrence
        if (gt == 0) {
          exact[set] = 1;
          mbar_arrive(bar_g + 8 * set);
        }
        continue;
      }
      if (gt == 0) exact[set] = 0;
      // ---- Q~ = q x and K~ = k / x in place, Khat = K~ e^{b_last - b_m} in its buffer
      {
        const float* X = reinterpret_cast<const float*>(sset + kSetA);
        const int c16 = gt & 15, col = c16 * 8;            // the same 8 channels in every item
        const float4 l0 = *reinterpret_cast<const float4*>(lam_r + col);
        const float4 l1 = *reinterpret_cast<const float4*>(lam_r + col + 4);
        const float ls[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
#pragma unroll
        for (int it = 0; it < L * 16 / kGroup; ++it) {
          const int r = (gt + it * kGroup) >> 4;
          const uint32_t off = swz(L, r, c16);
          const uint4 qv = *reinterpret_cast<const uint4*>(sset + kSetQ + off);
          const uint4 kv = *reinterpret_cast<const uint4*>(sset + kSetK + off);
          const float4 x0 = *reinterpret_cast<const float4*>(X + r * DK + col);
          const float4 x1 = *reinterpret_cast<const float4*>(X + r * DK + col + 4);
          const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          const uint32_t* qw = reinterpret_cast<const uint32_t*>(&qv);
          const uint32_t* kw = reinterpret_cast<const uint32_t*>(&kv);
          uint32_t qo[4], ko[4], ho[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 q2 = *reinterpret_cast<const __nv_bfloat162*>(&qw[e]);
            const __nv_bfloat162 k2 = *reinterpret_cast<const __nv_bfloat162*>(&kw[e]);
            const float ka = __low2float(k2) * rcp_approx(xs[2 * e]);
            const float kb = __high2float(k2) * rcp_approx(xs[2 * e + 1]);
            qo[e] = pack2(__low2float(q2) * xs[2 * e], __high2float(q2) * xs[2 * e + 1]);
            ko[e] = pack2(ka, kb);
            ho[e] = pack2(ka * ls[2 * e], kb * ls[2 * e + 1]);
          }
          *reinterpret_cast<uint4*>(sset + kSetQ + off) = make_uint4(qo[0], qo[1], qo[2], qo[3]);
          *reinterpret_cast<uint4*>(sset + kSetK + off) = make_uint4(ko[0], ko[1], ko[2], ko[3]);
          *reinterpret_cast<uint4*>(sset + kSetKhat + off) = make_uint4(ho[0], ho[1], ho[2], ho[3]);
        }
      }
      fence_proxy_async();                                 // generic writes -> tensor-core reads
      group_sync(kBarGate, kGroup);
      if (gt == 0) mbar_arrive(bar_g + 8 * set);           // chunk c is ready for the TMEM group
    }
  } else {
    // ================================================================ TMEM group
    const int quad = warp & 3, hc = warp >> 2;             // lane quadrant, column half
    const int row = quad * 32 + lane;                      // TMEM lane of this thread
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    // the initial state into TMEM: lane i holds value channel i (columns 64 hc .. + 63 here)
#pragma unroll 1
    for (int c0 = hc * 64; c0 < hc * 64 + 64; c0 += 32) {
      const float4* src = reinterpret_cast<const float4*>(st + (long long)row * DK + c0);
      uint32_t r[32];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float4 x = src[e];
        r[4 * e] = __float_as_uint(x.x); r[4 * e + 1] = __float_as_uint(x.y);
        r[4 * e + 2] = __float_as_uint(x.z); r[4 * e + 3] = __float_as_uint(x.w);
      }
      tmem_st32(lane_addr + kColS + c0, r);
    }
    tmem_wait_st();
    const uint32_t id_a = idesc2(64, 64, false, false);    // A = Q~ K~^T
    const uint32_t id_av = idesc2(64, DV, false, true);    // O += A V      (V: N-contiguous)
    const uint32_t id_qs = idesc2(64, DV, false, false);   // O += Q~ S_0'^T
    const uint32_t id_s = idesc2(128, DK, true, true);     // S += V^T Khat (both MN-contiguous)
    int phase = 0;
    for (int c = 0; c < n_chunks; ++c) {
      const int set = c & 1;
      const uint32_t sb = s0 + set * kSet;
      const float* lam_m = reinterpret_cast<const float*>(sm + kLam + set * 2 * DK * 4);
      const float* lam_r = lam_m + DK;
      ok = mbar_wait_bounded(bar_g + 8 * set, (c >> 1) & 1, kWait, abort_flag, nullptr, 0);
      if (tid == 0) bulk_wait_read();                      // the previous output tile has left S_0'
      if (!(ok = group_and(kBarTmem, kGroup, ok))) break;

      if (exact[set]) {
        // ---- the recurrence, token by token, on raw q, k, v and gates: this
        // thread holds S[row, 64 hc .. + 63] (in local memory: the loop over its
        // 16-byte chunks is not unrolled, to keep the main path's registers
        // free -- this path only runs for chunks with extreme gates); the half hc = 1 hands
        // its part of o_t[row] to hc = 0 through the set's (unused) Khat buffer,
        // which writes o_t as bf16 into the staging tile
        const uint8_t* sset = sm + set * kSet;
        float* xbuf = reinterpret_cast<float*>(sm + set * kSet + kSetKhat);   // [2][128]
        // the raw gates of this chunk (the shared table holds the factors)
        const float* a_chunk = a_raw + (((long long)b * T + (long long)c * L) * H + hd) * DK + hc * 64;
        float S[64];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t r[32];
          tmem_ld32(lane_addr + kColS + hc * 64 + 32 * h2, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) S[32 * h2 + e] = __uint_as_float(r[e]);
        }
#pragma unroll 1
        for (int t = 0; t < L; ++t) {
          const float* at = a_chunk + (long long)t * H * DK;
          const uint32_t vo = swz(L, t, row >> 3) + (row & 7) * 2;
          const float vt = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sset + kSetV + vo));
          float o = 0.f;
#pragma unroll 1
          for (int e8 = 0; e8 < 8; ++e8) {                 // 16-byte chunk hc * 8 + e8 of row t
            const uint32_t off = swz(L, t, hc * 8 + e8);
            const uint4 kv = *reinterpret_cast<const uint4*>(sset + kSetK + off);
            const uint4 qv = *reinterpret_cast<const uint4*>(sset + kSetQ + off);
            const float4 a0 = __ldg(reinterpret_cast<const float4*>(at + 8 * e8));
            const float4 a1 = __ldg(reinterpret_cast<const float4*>(at + 8 * e8 + 4));
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const uint32_t* kw = reinterpret_cast<const uint32_t*>(&kv);
            const uint32_t* qw = reinterpret_cast<const uint32_t*>(&qv);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 k2 = *reinterpret_cast<const __nv_bfloat162*>(&kw[e]);
              const __nv_bfloat162 q2 = *reinterpret_cast<const __nv_bfloat162*>(&qw[e]);
              float& s0v = S[8 * e8 + 2 * e];
              float& s1v = S[8 * e8 + 2 * e + 1];
              s0v = fmaf(s0v, av[2 * e], vt * __low2float(k2));
              s1v = fmaf(s1v, av[2 * e + 1], vt * __high2float(k2));
              o = fmaf(s0v, __low2float(q2), o);
              o = fmaf(s1v, __high2float(q2), o);
            }
          }
          if (hc == 1) xbuf[(t & 1) * DV + row] = o;
          group_sync(kBarTmem, kGroup);
          if (hc == 0) {
            o += xbuf[(t & 1) * DV + row];
            *reinterpret_cast<__nv_bfloat16*>(sm + kSb + vo) = __float2bfloat16_rn(o);
          }
        }
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t r[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(S[32 * h2 + e]);
          tmem_st32(lane_addr + kColS + hc * 64 + 32 * h2, r);
        }
        tmem_wait_st();
        fence_proxy_async();                               // staged rows -> the TMA store
        tc_fence_before();
        if (!(ok = group_and(kBarTmem, kGroup, ok))) break;   // the set has been read
        if (tid == 0) {
          tc_fence_after();
          if (c + 2 < n_chunks) {
            load_chunk(c + 2);
            ++n_issued;
          }
          tma_store_4d(&tm_o, s0 + kSb, 0, hd, c * L, b);
          tma_store_4d(&tm_o, s0 + kSb + kHalf, 64, hd, c * L, b);
          bulk_commit();
        }
        continue;
      }

      // ---- A = Q~ K~^T (64 x 64, K = 128) into the 64-row accumulator
      if (tid == 0) {
        tc_fence_after();
        const uint64_t dq = sdesc(sb + kSetQ, 16, 1024), dk = sdesc(sb + kSetK, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t off = ((ks >> 2) * kHalf + (ks & 3) * 32) >> 4;
          mma_f16(tmem + kColAO, dq + off, dk + off, id_a, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar_mma);
      }
      // ---- meanwhile S_0 -> its bf16 copy S_0 diag(e^{b_m}) (row = value
      // channel) and S_0 diag(e^{b_last}) back into TMEM (columns 64 hc .. + 63)
#pragma unroll 1
      for (int c0 = hc * 64; c0 < hc * 64 + 64; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lane_addr + kColS + c0, r);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(lam_m + c0 + e);
          const float4 r4 = *reinterpret_cast<const float4*>(lam_r + c0 + e);
          const float x0 = __uint_as_float(r[e]) * m4.x, x1 = __uint_as_float(r[e + 1]) * m4.y;
          const float x2 = __uint_as_float(r[e + 2]) * m4.z, x3 = __uint_as_float(r[e + 3]) * m4.w;
          pk[e / 2] = pack2(x0, x1);
          pk[e / 2 + 1] = pack2(x2, x3);
          r[e] = __float_as_uint(x0 * r4.x);
          r[e + 1] = __float_as_uint(x1 * r4.y);
          r[e + 2] = __float_as_uint(x2 * r4.z);
          r[e + 3] = __float_as_uint(x3 * r4.w);
        }
        tmem_st32(lane_addr + kColS + c0, r);
#pragma unroll
        for (int e = 0; e < 4; ++e)                       // 16-byte chunks (c0 / 8 + e) of this row
          *reinterpret_cast<uint4*>(sm + kSb + swz(DV, row, c0 / 8 + e)) =
              make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
      }
      tmem_wait_st();
      // ---- A: causal mask, bf16 -> shared over the set's consumed gate table
      // (row t = 16 quad + lane on lanes 0-15; columns 32 hc .. + 31)
      ok = mbar_wait_bounded(bar_mma, phase & 1, kWait, abort_flag, nullptr, 0);
      ++phase;
      tc_fence_after();
      {
        uint32_t r[32];
        tmem_ld32(lane_addr + kColAO + hc * 32, r);
        tmem_wait_ld();
        if (lane < 16) {
          const int t = quad * 16 + lane;
#pragma unroll
          for (int e = 0; e < 4; ++e) {                    // 16-byte chunk 4 hc + e
            uint32_t w[4];
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              const int cc = 8 * e + 2 * f, s = hc * 32 + cc;
              w[f] = pack2(s <= t ? __uint_as_float(r[cc]) : 0.f, s + 1 <= t ? __uint_as_float(r[cc + 1]) : 0.f);
            }
            const int ch = hc * 4 + e;
            *reinterpret_cast<uint4*>(sm + set * kSet + kSetA + t * 128 + ((ch ^ (t & 7)) << 4)) =
                make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      fence_proxy_async();
      tc_fence_before();
      if (!(ok = group_and(kBarTmem, kGroup, ok))) break;

      // ---- O = A V + Q~ S_0'^T (64 x 128) and S += V^T Khat (128 x 128)
      if (tid == 0) {
        tc_fence_after();
        const uint64_t dab = sdesc(sb + kSetA, 16, 1024);
        const uint64_t dv_b = sdesc(sb + kSetV, kHalf, 1024);      // V as N-contiguous B
        const uint64_t dq = sdesc(sb + kSetQ, 16, 1024), dsb = sdesc(s0 + kSb, 16, 1024);
        const uint64_t dv_a = sdesc(sb + kSetV, kHalf, 1024);      // V^T as M-contiguous A
        const uint64_t dkh = sdesc(sb + kSetKhat, kHalf, 1024);    // Khat as N-contiguous B
#pragma unroll
        for (int ks = 0; ks < L / 16; ++ks)
          mma_f16(tmem + kColAO, dab + ((ks * 32) >> 4), dv_b + ((ks * 2048) >> 4), id_av,
                  ks > 0 ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t offq = ((ks >> 2) * kHalf + (ks & 3) * 32) >> 4;
          const uint32_t offs = ((ks >> 2) * (DV * 128) + (ks & 3) * 32) >> 4;
          mma_f16(tmem + kColAO, dq + offq, dsb + offs, id_qs, 1u);
        }
#pragma unroll
        for (int ks = 0; ks < L / 16; ++ks)
          mma_f16(tmem + kColS, dv_a + ((ks * 2048) >> 4), dkh + ((ks * 2048) >> 4), id_s, 1u);
        mma_commit(bar_mma);
      }
      ok = mbar_wait_bounded(bar_mma, phase & 1, kWait, abort_flag, nullptr, 0);
      ++phase;
      tc_fence_after();
      // the set is free: chunk c + 2's inputs start loading into it
      if (tid == 0 && ok && c + 2 < n_chunks) {
        load_chunk(c + 2);
        ++n_issued;
      }
      // ---- O -> bf16 rows (row t = 16 quad + lane on lanes 0-15; columns
      // 64 hc .. + 63), staged as a [64][128] 128B-swizzled tile in the S_0'
      // buffer (free until the next state pass), then one TMA store per half;
      // thread 0 waits for the store to have read it before that pass
#pragma unroll 1
      for (int c0 = hc * 64; c0 < hc * 64 + 64; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lane_addr + kColAO + c0, r);
        tmem_wait_ld();
        if (lane < 16) {
          const int t = quad * 16 + lane;
#pragma unroll
          for (int e = 0; e < 4; ++e)
            *reinterpret_cast<uint4*>(sm + kSb + swz(L, t, c0 / 8 + e)) =
                make_uint4(pack2(__uint_as_float(r[8 * e]), __uint_as_float(r[8 * e + 1])),
                           pack2(__uint_as_float(r[8 * e + 2]), __uint_as_float(r[8 * e + 3])),
                           pack2(__uint_as_float(r[8 * e + 4]), __uint_as_float(r[8 * e + 5])),
                           pack2(__uint_as_float(r[8 * e + 6]), __uint_as_float(r[8 * e + 7])));
        }
      }
      fence_proxy_async();                                 // staged rows -> the TMA store
      tc_fence_before();
      if (!(ok = group_and(kBarTmem, kGroup, ok))) break;  // the accumulator is reused next
      if (tid == 0) {
        tma_store_4d(&tm_o, s0 + kSb, 0, hd, c * L, b);
        tma_store_4d(&tm_o, s0 + kSb + kHalf, 64, hd, c * L, b);
        bulk_commit();
      }
    }
    if (!ok && tid == 0) {                                 // MMAs in flight end before exit
      mma_commit(bar_mma);
      const unsigned long long t_m = global_ns();
      while (!mbar_try_wait_parity(bar_mma, phase & 1) && global_ns() - t_m < kWait) {
      }
    }
    // ---- the final state (NaN if a wait ran out): columns 64 hc .. + 63 of this lane
    tc_fence_after();
#pragma unroll 1
    for (int c0 = hc * 64; c0 < hc * 64 + 64; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(lane_addr + kColS + c0, r);
      tmem_wait_ld();
      float4* dst = reinterpret_cast<float4*>(st + (long long)row * DK + c0);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        dst[e] = ok ? make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                  __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]))
                    : make_float4(NAN, NAN, NAN, NAN);
    }
  }
  // copies in flight land before exit (the last two requested sets; a set that
  // was consumed reads as complete)
  if (tid == 0 && *abort_flag) {
    for (int i = n_issued - 2 > 0 ? n_issued - 2 : 0; i < n_issued; ++i) {
      const unsigned long long t_0 = global_ns();
      while (!mbar_try_wait_parity(bar_in + 8 * (i & 1), (i >> 1) & 1) && global_ns() - t_0 < kWait) {
      }
    }
  }
  if (tid == 0) bulk_wait_all();                         // output stores complete before exit
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace glatc

cudaError_t gla_prefill_tc(int B, int T, int H, const void* q, const void* k, const void* v,
                           const float* a, void* o, float* state, cudaStream_t stream) {
  using namespace glatc;
  CUtensorMap mq, mk, mv, ma, mo;
  const cuuint64_t dims[4] = {(cuuint64_t)DK, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t sb[3] = {(cuuint64_t)DK * 2, (cuuint64_t)H * DK * 2, (cuuint64_t)T * H * DK * 2};
  const cuuint64_t sf[3] = {(cuuint64_t)DK * 4, (cuuint64_t)H * DK * 4, (cuuint64_t)T * H * DK * 4};
  const cuuint32_t box_b[4] = {64, 1, (cuuint32_t)L, 1}, box_f[4] = {(cuuint32_t)DK, 1, (cuuint32_t)L, 1};
  if (!tc::encode(&mq, q, 4, dims, sb, box_b) || !tc::encode(&mk, k, 4, dims, sb, box_b) ||
      !tc::encode(&mv, v, 4, dims, sb, box_b) || !tc::encode(&mo, o, 4, dims, sb, box_b) ||
      !tc::encode_ex(&ma, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, CU_TENSOR_MAP_SWIZZLE_NONE, a, 4, dims,
                     sf, box_f))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(gla_prefill_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  gla_prefill_tc_kernel<<<B * H, kThreads, kSmem, stream>>>(mq, mk, mv, ma, mo, T, H, a, state);
  return cudaGetLastError();
}

}  // namespace lte
