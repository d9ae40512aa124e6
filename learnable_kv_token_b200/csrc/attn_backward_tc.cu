// dQ of the prefill sparse attention's backward on 5th-generation tensor
// cores (tcgen05 + TMEM), head dim 128, bf16 operands, fp32 accumulation.
//
// "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention
// and Contextualized Learnable Token Eviction", Abstract (trained end to end)
// and Fig. 2 caption (right): the attended sets S_t, held fixed.  Per query
// row, with P recomputed from the forward's lse and D_t = <dO_t, o_t>:
//   dS = P * (dO V^T - D_t),   dQ = scale dS K.
//
// One CTA of 128 threads per 128 query rows (128/G tokens x the G heads of a
// KV head, token-major), one row per thread; two CTAs share an SM (112 KiB of
// shared memory and 256 TMEM columns each).  Q and dO stay in shared memory;
// per 64-key tile of the forward's key ranges (sink slots and retained slots
// of the column segment, window band of k):
//   1. K and V of the tile arrive by cp.async (zero-filled past the tile's
//      valid rows) in the 128-byte-swizzled K-major layout;
//   2. one thread issues S = Q K^T and dP = dO V^T (M128 N64 K128, both
//      operands in shared memory) into TMEM and commits;
//   3. each thread reads its row of S and dP, forms P (masked keys 0) and
//      dS = P (dP - D_t), and writes dS as bf16 into shared memory (the A
//      operand of the next product);
//   4. one thread issues dQ += dS K (M128 N128 K64; K as an N-contiguous B
//      operand) into the TMEM accumulator and commits; the tile's buffers are
//      reused once that product has completed.
// Every wait is bounded; on expiry the CTA records LTE_ERR_TIMEOUT, drains
// what it issued, frees its TMEM and leaves.
#include <math.h>

#include "attn_backward.cuh"
#include "lte_common.cuh"
#include "lte_internal.h"
#include "tc_ptx.cuh"

namespace lte {
namespace bwdtc {

using namespace tc;

constexpr int HD = 128;
constexpr int kRowsTc = 128;                    // query rows per CTA
constexpr int kKeysTc = 64;                     // keys per tile
constexpr int kThreadsTc = 128;
constexpr uint32_t kQ = 0;                      // [128][128] bf16: two 64-column halves of 16 KiB
constexpr uint32_t kDO = 32768;                 // same for dO
constexpr uint32_t kK = 65536;                  // [64][128]: two halves of 8 KiB
constexpr uint32_t kV = 81920;
constexpr uint32_t kDS = 98304;                 // [128][64] bf16 (one half)
constexpr uint32_t kBar = 114688;               // bar_s, bar_q, abort flag, TMEM slot
constexpr int kSmemBytes = kBar + 64;
constexpr int kTmemCols = 256;                  // S 0..63, dP 64..127, dQ 128..255
constexpr uint32_t kColS = 0, kColDP = 64, kColDQ = 128;

// byte offset of 16-byte chunk c16 (0..15) of row r in a K-major [rows][128]
// bf16 tile stored as two 64-column halves, 128-byte swizzle
__device__ __forceinline__ uint32_t sw(int rows, int r, int c16) {
  return (uint32_t)((c16 >> 3) * rows * 128 + r * 128 + ((((c16 & 7) ^ (r & 7))) << 4));
}
__device__ __forceinline__ void cpa16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cpa_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cpa_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::); }
// bits [a, b) of a 64-bit set (empty when b <= a), clipped to [0, 64)
__device__ __forceinline__ uint64_t span64(int a, int b) {
  a = a > 0 ? a : 0;
  b = b < 64 ? b : 64;
  if (b <= a) return 0ull;
  const uint64_t ones = (b - a == 64) ? ~0ull : ((1ull << (b - a)) - 1ull);
  return ones << a;
}
// first index i in [0, n) with v[i] > x for a nondecreasing v (n if none)
__device__ __forceinline__ int first_above(const int* v, int n, int x) {
  int l = 0, r = n;
  while (l < r) {
    const int m = (l + r) >> 1;
    if (v[m] > x) r = m; else l = m + 1;
  }
  return l;
}
__device__ __forceinline__ uint32_t pk2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Pipelined roles (256 threads, one CTA per SM):
//   warp 0     TMA copies (one elected lane): Q and dO once, then K and V of key
//              tile j into ring stage j % 3 (128-byte swizzled 64-column halves;
//              rows past the tensor read as zero);
//   warp 1     issues, per tile j: S(j), dP(j) into TMEM buffer j % 2, then
//              dQ += dS(j-1) K(j-1) once dS(j-1) is in shared memory -- so the
//              tensor core computes tile j's products while the rows of tile
//              j - 1 are being formed;
//   warps 4-11 two threads per query row (warps 4-7 the first 32 keys of a
//              tile, 8-11 the last 32): P and dS of tile j from TMEM buffer
//              j % 2 into the shared dS buffer j % 2; at the end, dQ out (64
//              of the 128 columns each).  Two warps per sub-partition hide
//              each other's TMEM and special-function latency.
// TMEM: S[2] 0..127, dP[2] 128..255, dQ 256..383.
constexpr int kThreadsP = 384;
constexpr int kStagesP = 3;                             // K/V ring
constexpr uint32_t kK2 = 65536;                         // stage s: K at + 32 KiB s, V at + 16 KiB
constexpr uint32_t kDS2 = kK2 + kStagesP * 32768;       // dS buffers: 2 x [128][64] bf16
constexpr uint32_t kBar2 = kDS2 + 2 * 16384;            // barriers
constexpr int kSmemP = kBar2 + 256;
constexpr uint32_t kColSP = 0, kColDPP = 128, kColDQP = 256;
enum {
  P_QF = 0, P_KVF = 1, P_KVE = P_KVF + kStagesP, P_SF = P_KVE + kStagesP, P_SE = P_SF + 2,
  P_DSF = P_SE + 2, P_DSE = P_DSF + 2, P_DQ = P_DSE + 2, kNumBarsP = P_DQ + 1
};
static_assert(8 * kNumBarsP + 8 <= 256, "barriers fit");

__global__ void __launch_bounds__(kThreadsP, 1)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc,
                 const bwd::Args a, DevError* err) {
  extern __shared__ __align__(1024) uint8_t sm[];
  const uint32_t sb = sa(sm);
  if ((sb & 1023u) != 0) {                      // swizzle atoms need 1 KiB alignment
    if (threadIdx.x == 0) record_error(err, LTE_ERR_DEVICE, 403);
    return;
  }
  auto bar = [&](int i) { return sb + kBar2 + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kBar2 + 8 * kNumBarsP);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kBar2 + 8 * kNumBarsP + 4);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int G = a.G, TOK = kRowsTc / G;
  const int n_tiles = (a.T + TOK - 1) / TOK;
  const int t0 = (n_tiles - 1 - (int)blockIdx.x) * TOK;          // late (heavy) tiles first
  const int h = blockIdx.y, b = blockIdx.z, u = b * a.Hkv + h;
  const int t_last = min(t0 + TOK - 1, a.T - 1);
  const long long crow = (long long)u * a.T;
  const long long col_base = (long long)u * (a.sink + a.T);
  const bool lowest = a.death != nullptr;

  if (tid == 0) {
    mbar_init(bar(P_QF), 1);
    for (int x = 0; x < kStagesP; ++x) {
      mbar_init(bar(P_KVF + x), 1);
      mbar_init(bar(P_KVE + x), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(P_SF + x), 1);
      mbar_init(bar(P_SE + x), 256);
      mbar_init(bar(P_DSF + x), 256);
      mbar_init(bar(P_DSE + x), 1);
    }
    mbar_init(bar(P_DQ), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     sa(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // key ranges of the tile: 0 sink slots, 1 retained slots, 2 window band
  int start[3], count[3];
  {
    int lo_f, n_first, lo_l, n_last;
    bwd::row_range(a, crow, t0, lo_f, n_first);
    bwd::row_range(a, crow, t_last, lo_l, n_last);
    const int lo_min = lowest ? 0 : lo_f;
    int nsink = t_last - a.window + 1;
    nsink = nsink < 0 ? 0 : (nsink > a.sink ? a.sink : nsink);
    nsink = nsink > a.T ? a.T : nsink;
    const int w_lo = t0 - a.window + 1 > 0 ? t0 - a.window + 1 : 0;
    start[0] = 0; count[0] = nsink;
    start[1] = a.sink + lo_min; count[1] = (a.cap > 0 && n_last > lo_min) ? n_last - lo_min : 0;
    start[2] = w_lo; count[2] = t_last - w_lo + 1;
  }
  const int n0 = (count[0] + kKeysTc - 1) / kKeysTc, n1 = (count[1] + kKeysTc - 1) / kKeysTc;
  const int total = n0 + n1 + (count[2] + kKeysTc - 1) / kKeysTc;
  auto tile_of = [&](int j, int& rg, int& key0, int& nk) {
    int it = j;
    if (it < n0) rg = 0;
    else if (it < n0 + n1) { rg = 1; it -= n0; }
    else { rg = 2; it -= n0 + n1; }
    key0 = start[rg] + it * kKeysTc;
    nk = min(kKeysTc, count[rg] - it * kKeysTc);
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    bool ok = true;
    if (elect_one()) {
      mbar_expect_tx(bar(P_QF), 2 * kRowsTc * HD * 2);
      for (int hf = 0; hf < 2; ++hf) {
        tma_load_4d(sb + kQ + hf * (kRowsTc * 128), &tm_q, bar(P_QF), hf * 64, h * G, t0, b);
        tma_load_4d(sb + kDO + hf * (kRowsTc * 128), &tm_do, bar(P_QF), hf * 64, h * G, t0, b);
      }
    }
    __syncwarp();
    int issued = 0;
    for (int j = 0; j < total && ok; ++j) {
      const int st = j % kStagesP, use = j / kStagesP;
      if (use >= 1 && !(ok = wwait(bar(P_KVE + st), (use - 1) & 1, abort_flag, err, 404))) break;
      int rg, key0, nk;
      tile_of(j, rg, key0, nk);
      if (elect_one()) {
        const uint32_t kd = sb + kK2 + st * 32768u, vd = kd + 16384u;
        mbar_expect_tx(bar(P_KVF + st), 2 * kKeysTc * HD * 2);
        for (int hf = 0; hf < 2; ++hf) {
          if (rg == 2) {
            tma_load_4d(kd + hf * (kKeysTc * 128), &tm_k, bar(P_KVF + st), hf * 64, h, key0, b);
            tma_load_4d(vd + hf * (kKeysTc * 128), &tm_v, bar(P_KVF + st), hf * 64, h, key0, b);
          } else {
            tma_load_3d(kd + hf * (kKeysTc * 128), &tm_kc, bar(P_KVF + st), hf * 64, key0, u);
            tma_load_3d(vd + hf * (kKeysTc * 128), &tm_vc, bar(P_KVF + st), hf * 64, key0, u);
          }
        }
      }
      __syncwarp();
      issued = j + 1;
    }
    // every issued copy has landed before the CTA may exit
    mbar_drain(bar(P_QF), 0);
    for (int q = issued - kStagesP > 0 ? issued - kStagesP : 0; q < issued; ++q)
      mbar_drain(bar(P_KVF + q % kStagesP), (q / kStagesP) & 1);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t id_s = idesc(kRowsTc, kKeysTc, false);     // S, dP: K-major A and B
    const uint32_t id_q = idesc(kRowsTc, HD, true);           // dQ: K as an N-contiguous B
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar(P_QF), 0, abort_flag, err, 405));
    auto issue_dq = [&](int jj) -> bool {                     // dQ += dS(jj) K(jj)
      const int x = jj & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(P_DSF + x), (jj >> 1) & 1, abort_flag, err, 406)))
        return false;
      tc_fence_after();
      if (elect_one()) {
        const uint64_t dds = sdesc(sb + kDS2 + x * 16384u, 16, 1024);
        const uint64_t dkb = sdesc(sb + kK2 + (jj % kStagesP) * 32768u, kKeysTc * 128, 1024);
#pragma unroll
        for (int ks = 0; ks < kKeysTc / 16; ++ks)
          mma_f16(tmem + kColDQP, dds + ((ks * 32) >> 4), dkb + ((ks * 2048) >> 4), id_q,
                  (jj > 0 || ks > 0) ? 1u : 0u);
        mma_commit(bar(P_DSE + x));                           // dS buffer x is free
        mma_commit(bar(P_KVE + jj % kStagesP));               // K, V of tile jj are free
      }
      __syncwarp();
      return true;
    };
    for (int j = 0; j < total && ok; ++j) {
      const int x = j & 1, use = j >> 1, st = j % kStagesP;
      ok = mbar_wait(bar(P_KVF + st), (j / kStagesP) & 1, abort_flag, err, 407);
      if (ok && use >= 1) ok = mbar_wait(bar(P_SE + x), (use - 1) & 1, abort_flag, err, 408);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      if (elect_one()) {
        const uint64_t dq_ = sdesc(sb + kQ, 16, 1024), ddo = sdesc(sb + kDO, 16, 1024);
        const uint64_t dk = sdesc(sb + kK2 + st * 32768u, 16, 1024);
        const uint64_t dv = sdesc(sb + kK2 + st * 32768u + 16384u, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
          const uint32_t oa = ((ks >> 2) * (kRowsTc * 128) + (ks & 3) * 32) >> 4;
          const uint32_t ob = ((ks >> 2) * (kKeysTc * 128) + (ks & 3) * 32) >> 4;
          mma_f16(tmem + kColSP + x * 64, dq_ + oa, dk + ob, id_s, ks > 0 ? 1u : 0u);
          mma_f16(tmem + kColDPP + x * 64, ddo + oa, dv + ob, id_s, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar(P_SF + x));
      }
      __syncwarp();
      if (j >= 1 && !(ok = issue_dq(j - 1))) break;
    }
    if (ok && total > 0) ok = issue_dq(total - 1);
    if (elect_one()) mma_commit(bar(P_DQ));                   // every product above has completed
    __syncwarp();
    mbar_drain(bar(P_DQ), 0);
  } else {
    // ---------------------------------------------------------------- rows (warps 4-11)
    if (warp < 4) {
      // warps 2-3 have no role
    } else {
    const int quad = warp & 3, kh = (warp - 4) >> 2;   // TMEM lane quadrant, key half of a tile
    const int row = quad * 32 + (tid & 31);
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const int tt = t0 + row / G, gq = row % G;
    int lo_r, hi_r;
    bwd::row_range(a, crow, tt, lo_r, hi_r);
    if (lowest) lo_r = 0;
    float lse2 = 0.f, dl = 0.f;
    if (tt < a.T) {
      const long long li = ((long long)b * a.Hq + h * G + gq) * a.T + tt;
      lse2 = a.lse[li] * 1.4426950408889634f;
      dl = a.delta[li];
    }
    bool ok = true;
    for (int j = 0; j < total && ok; ++j) {
      const int x = j & 1, use = j >> 1;
      int rg, key0, nk;
      tile_of(j, rg, key0, nk);
      // this row's keys in the tile: at most two intervals (sink slots, retained
      // slots [lo, hi)) or one (window band); this thread takes keys 32 kh ..
      uint64_t bits = 0ull;
      if (tt < a.T) {
        if (rg == 2) {
          bits = span64(tt - a.window + 1 - key0, min(nk, tt - key0 + 1));
        } else {
          const int sink_end = min(a.sink, tt - a.window + 1);
          uint64_t ret = span64(a.sink + lo_r - key0, min(nk, a.sink + hi_r - key0));
          if (lowest && ret != 0ull) {                 // lifetimes: held at count hi_r
#pragma unroll 4
            for (int kk = 32 * kh; kk < 32 * kh + 32; ++kk)
              if (((ret >> kk) & 1ull) && __ldg(a.death + crow + key0 + kk - a.sink) <= hi_r)
                ret &= ~(1ull << kk);
          }
          bits = span64(-key0, min(nk, sink_end - key0)) | ret;
        }
      }
      const uint32_t hb = (uint32_t)(bits >> (32 * kh));
      const float* brow = (a.bias != nullptr && rg != 2) ? a.bias + col_base + key0 + 32 * kh : nullptr;
      ok = mbar_wait(bar(P_SF + x), use & 1, abort_flag, err, 409);
      if (ok && use >= 1) ok = mbar_wait(bar(P_DSE + x), (use - 1) & 1, abort_flag, err, 410);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      uint32_t pkd[16];
      {
        uint32_t rs[32], rp[32];
        tmem_ld32(lane_addr + kColSP + x * 64 + 32 * kh, rs);
        tmem_ld32(lane_addr + kColDPP + x * 64 + 32 * kh, rp);
        tmem_wait_ld();
        if (brow != nullptr) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if ((hb >> c) & 1u) rs[c] = __float_as_uint(__uint_as_float(rs[c]) + __ldg(brow + c));
        }
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float ds2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float p = ((hb >> (c + e)) & 1u)
                                ? ex2(fmaf(__uint_as_float(rs[c + e]), a.scale_log2, -lse2))
                                : 0.f;
            ds2[e] = p * (__uint_as_float(rp[c + e]) - dl);
          }
          pkd[c >> 1] = pk2(ds2[0], ds2[1]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(P_SE + x));                      // this thread's part of S, dP x is read
      // 64 bytes of the dS row (keys 32 kh ..) into the swizzled K-major A operand
      uint8_t* drow = sm + kDS2 + x * 16384u + row * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int ch = 4 * kh + c;
        *reinterpret_cast<uint4*>(drow + ((ch ^ (row & 7)) << 4)) =
            make_uint4(pkd[4 * c], pkd[4 * c + 1], pkd[4 * c + 2], pkd[4 * c + 3]);
      }
      fence_proxy_async();
      mbar_arrive(bar(P_DSF + x));
    }
    // dQ row: scale, fp32 out, columns 64 kh .. (every lane loads: tcgen05.ld is warp-collective)
    ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(P_DQ), 0, abort_flag, err, 411));
    if (ok) {
      tc_fence_after();
      float* out = a.dq + (((long long)b * a.T + min(tt, a.T - 1)) * a.Hq + h * G + gq) * HD;
#pragma unroll 1
      for (int c0 = 64 * kh; c0 < 64 * kh + 64; c0 += 32) {
        uint32_t r[32];
        if (total > 0) {
          tmem_ld32(lane_addr + kColDQP + c0, r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = 0u;
        }
        if (tt < a.T) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(out + c0 + e) =
                make_float4(__uint_as_float(r[e]) * a.scale, __uint_as_float(r[e + 1]) * a.scale,
                            __uint_as_float(r[e + 2]) * a.scale, __uint_as_float(r[e + 3]) * a.scale);
        }
      }
    }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                 : "memory");
}

// ---------------------------------------------------------------- dK, dV
// One CTA per 128-key tile (keys of k for the window part, kColumn = false;
// slots of the column segment, kColumn = true, for this CTA's share of the
// attending rows).  Keys are the MMA rows; the attending query rows come in
// tiles of 64 (64/G tokens x the G heads), and per row tile i:
//   S^T = K Q^T, dP^T = V dO^T        (M128 N64 K128) into TMEM buffer i % 2
//   P^T, dS^T = P^T (dP^T - D)         (two threads per key row, 32 rows each)
//   dV += P^T dO, dK += dS^T Q         (M128 N128 K64; P^T, dS^T read from TMEM)
// Roles (384 threads, one CTA per SM):
//   warp 0     TMA producer (one elected lane): K and V once; per row tile, Q
//              and dO into a 3-stage ring, the rows' lse, D, token and retained
//              range written by the warp's lanes into the stage;
//   warp 1     MMA issuer: S^T(i), dP^T(i), then dV and dK of tile i - 1 once
//              its P^T and dS^T are in TMEM -- the tensor core computes tile i
//              while the rows of tile i - 1 are formed;
//   warps 4-11 two threads per key row (warps 4-7 rows 0-31 of a tile, 8-11
//              rows 32-63): P^T and dS^T, written as bf16 over their own
//              columns of S^T and dP^T; at the end, dK and dV out.
// TMEM: S^T[2] 0..127, dP^T[2] 128..255, dV 256..383, dK 384..511.
constexpr int kKeysKV = 128;
constexpr int kRowsK2 = 64;                       // attending query rows per tile
constexpr int kStagesK2 = 3;
constexpr int kThreadsK2 = 384;
constexpr int kSplitRowsK2 = 32;                  // row tiles per CTA of the column pass
constexpr uint32_t k2K = 0, k2V = 32768;          // [128][128] bf16: halves of 16 KiB
constexpr uint32_t k2QD = 65536;                  // stage s: Q at + 32 KiB s, dO at + 16 KiB
constexpr uint32_t k2Meta = k2QD + kStagesK2 * 32768;            // stage s: [5][64] words
constexpr uint32_t k2Bar = k2Meta + kStagesK2 * 5 * kRowsK2 * 4;
constexpr int k2Smem = k2Bar + 256;
enum {
  K2_KVF = 0, K2_F = 1, K2_E = K2_F + kStagesK2, K2_SF = K2_E + kStagesK2, K2_PF = K2_SF + 2,
  K2_DONE = K2_PF + 2, kNumBarsK2 = K2_DONE + 1
};
static_assert(8 * kNumBarsK2 + 16 <= 256, "barriers, flags and the row range fit");

template <bool kColumn>
__global__ void __launch_bounds__(kThreadsK2, 1)
bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const bwd::Args a, int n_split, DevError* err) {
  extern __shared__ __align__(1024) uint8_t sm[];
  const uint32_t sb = sa(sm);
  if ((sb & 1023u) != 0) {
    if (threadIdx.x == 0) record_error(err, LTE_ERR_DEVICE, 413);
    return;
  }
  auto bar = [&](int i) { return sb + k2Bar + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + k2Bar + 8 * kNumBarsK2);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + k2Bar + 8 * kNumBarsK2 + 4);
  int* range_sh = reinterpret_cast<int*>(sm + k2Bar + 8 * kNumBarsK2 + 8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G, TOK = kRowsK2 / G;
  const int h = blockIdx.y, b = blockIdx.z, u = b * a.Hkv + h;
  const long long crow = (long long)u * a.T;
  const long long col_base = (long long)u * (a.sink + a.T);
  const bool lowest = a.death != nullptr;
  const int tile = kColumn ? (int)blockIdx.x / n_split : (int)blockIdx.x;
  const int split = kColumn ? (int)blockIdx.x % n_split : 0;
  const int k0 = tile * kKeysKV;
  const int nk = kColumn ? min(kKeysKV, a.sink + __ldg(a.nret + u) - k0) : min(kKeysKV, a.T - k0);
  if (nk <= 0) return;

  // row tiles that attend some key of this tile (this CTA's share of them)
  if (tid == 0) {
    int lo_t, hi_t;
    bwd::attending_tokens(a, crow, kColumn, k0, nk, lo_t, hi_t);
    int rt0 = lo_t / TOK, rt1 = hi_t / TOK;
    if (lo_t > hi_t) rt0 = 1, rt1 = 0;
    if constexpr (kColumn) {
      if (rt0 <= rt1) {
        const int first = rt0 + split * kSplitRowsK2;
        rt1 = min(rt1, first + kSplitRowsK2 - 1);
        rt0 = first;
      }
    }
    range_sh[0] = rt0;
    range_sh[1] = rt1;
  }
  __syncthreads();
  const int rt0 = range_sh[0], n_rt = range_sh[1] - range_sh[0] + 1;
  if (n_rt <= 0) return;                               // nothing attends (uniform)

  if (tid == 0) {
    mbar_init(bar(K2_KVF), 1);
    for (int st = 0; st < kStagesK2; ++st) {
      mbar_init(bar(K2_F + st), 1);
      mbar_init(bar(K2_E + st), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(K2_SF + x), 1);
      mbar_init(bar(K2_PF + x), 256);
    }
    mbar_init(bar(K2_DONE), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     sa(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    bool ok = true;
    if (elect_one()) {
      mbar_expect_tx(bar(K2_KVF), 2 * kKeysKV * HD * 2);
      for (int hf = 0; hf < 2; ++hf) {
        if constexpr (kColumn) {
          tma_load_3d(sb + k2K + hf * 16384u, &tm_k, bar(K2_KVF), hf * 64, k0, u);
          tma_load_3d(sb + k2V + hf * 16384u, &tm_v, bar(K2_KVF), hf * 64, k0, u);
        } else {
          tma_load_4d(sb + k2K + hf * 16384u, &tm_k, bar(K2_KVF), hf * 64, h, k0, b);
          tma_load_4d(sb + k2V + hf * 16384u, &tm_v, bar(K2_KVF), hf * 64, h, k0, b);
        }
      }
    }
    __syncwarp();
    int issued = 0;
    for (int i = 0; i < n_rt && ok; ++i) {
      const int st = i % kStagesK2, use = i / kStagesK2;
      if (use >= 1 && !(ok = wwait(bar(K2_E + st), (use - 1) & 1, abort_flag, err, 414))) break;
      // the rows' data: lse (log2), D, token, retained range [lo, hi)
      const int t0r = (rt0 + i) * TOK;
      float* mf = reinterpret_cast<float*>(sm + k2Meta) + st * 5 * kRowsK2;
      int* mi = reinterpret_cast<int*>(mf);
      for (int r = lane; r < kRowsK2; r += 32) {
        const int tt = t0r + r / G, g = r % G;
        float l2 = 0.f, dd = 0.f;
        int cv = 0;
        if (tt < a.T) {
          const long long li = ((long long)b * a.Hq + h * G + g) * a.T + tt;
          l2 = __ldg(a.lse + li) * 1.4426950408889634f;
          dd = __ldg(a.delta + li);
          if (tt >= a.window) cv = __ldg(a.cnt + crow + tt - a.window);
        }
        const int hi = (tt < a.T && tt >= a.window) ? held_retained(cv, a.cap, a.cap_policy) : 0;
        const int lo = (!lowest && a.cap_policy == LTE_CAP_RECENT && hi - a.cap > 0) ? hi - a.cap : 0;
        mf[r] = l2;
        mf[kRowsK2 + r] = dd;
        mi[2 * kRowsK2 + r] = tt;
        mi[3 * kRowsK2 + r] = lo;
        mi[4 * kRowsK2 + r] = hi;
      }
      __syncwarp();
      if (elect_one()) {
        const uint32_t qs = sb + k2QD + st * 32768u;
        mbar_expect_tx(bar(K2_F + st), 2 * kRowsK2 * HD * 2);
        for (int hf = 0; hf < 2; ++hf) {
          tma_load_4d(qs + hf * 8192u, &tm_q, bar(K2_F + st), hf * 64, h * G, t0r, b);
          tma_load_4d(qs + 16384u + hf * 8192u, &tm_do, bar(K2_F + st), hf * 64, h * G, t0r, b);
        }
      }
      __syncwarp();
      issued = i + 1;
    }
    // every issued copy has landed before the CTA may exit
    mbar_drain(bar(K2_KVF), 0);
    for (int q = issued - kStagesK2 > 0 ? issued - kStagesK2 : 0; q < issued; ++q)
      mbar_drain(bar(K2_F + q % kStagesK2), (q / kStagesK2) & 1);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t id_s = idesc(kKeysKV, kRowsK2, false);    // S^T, dP^T: K-major A and B
    const uint32_t id_o = idesc(kKeysKV, HD, true);          // dV, dK: dO, Q as N-contiguous B
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar(K2_KVF), 0, abort_flag, err, 415));
    auto issue_dvdk = [&](int i) -> bool {                   // dV, dK of row tile i
      const int x = i & 1, st = i % kStagesK2;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(K2_PF + x), (i >> 1) & 1, abort_flag, err, 416)))
        return false;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t qs = sb + k2QD + st * 32768u;
        const uint64_t qb = sdesc(qs, kRowsK2 * 128, 1024), dob = sdesc(qs + 16384u, kRowsK2 * 128, 1024);
#pragma unroll
        for (int ks = 0; ks < kRowsK2 / 16; ++ks) {
          // rows 16 ks .. of P^T, dS^T: the 32 rows of a thread pair's half sit in
          // columns 32 half .. + 15 of the buffer
          const uint32_t pc = (uint32_t)(x * 64 + 32 * (ks >> 1) + 8 * (ks & 1));
          const uint32_t acc = (i > 0 || ks > 0) ? 1u : 0u;
          mma_f16_ts(tmem + 256, tmem + pc, dob + ((ks * 2048) >> 4), id_o, acc);
          mma_f16_ts(tmem + 384, tmem + 128 + pc, qb + ((ks * 2048) >> 4), id_o, acc);
        }
        mma_commit(bar(K2_E + st));                          // the row tile's stage is free
      }
      __syncwarp();
      return true;
    };
    for (int i = 0; i < n_rt && ok; ++i) {
      const int x = i & 1, st = i % kStagesK2;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(K2_F + st), (i / kStagesK2) & 1, abort_flag, err, 417));
      if (!ok) break;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t qs = sb + k2QD + st * 32768u;
        const uint64_t dk = sdesc(sb + k2K, 16, 1024), dv = sdesc(sb + k2V, 16, 1024);
        const uint64_t dq = sdesc(qs, 16, 1024), ddo = sdesc(qs + 16384u, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
          const uint32_t oa = ((ks >> 2) * (kKeysKV * 128) + (ks & 3) * 32) >> 4;
          const uint32_t ob = ((ks >> 2) * (kRowsK2 * 128) + (ks & 3) * 32) >> 4;
          mma_f16(tmem + x * 64, dk + oa, dq + ob, id_s, ks > 0 ? 1u : 0u);
          mma_f16(tmem + 128 + x * 64, dv + oa, ddo + ob, id_s, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar(K2_SF + x));
      }
      __syncwarp();
      if (i >= 1 && !(ok = issue_dvdk(i - 1))) break;
    }
    if (ok) ok = issue_dvdk(n_rt - 1);
    if (elect_one()) mma_commit(bar(K2_DONE));             // every product above has completed
    __syncwarp();
    mbar_drain(bar(K2_DONE), 0);
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- key rows (warps 4-11)
    const int quad = warp & 3, half = (warp - 4) >> 2;     // TMEM lane quadrant, row half
    const int key_row = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const int kpos = k0 + key_row;                         // position (window) or slot (column)
    int kdeath = 0;
    if (kColumn && lowest && kpos >= a.sink && key_row < nk) kdeath = __ldg(a.death + crow + kpos - a.sink);
    // relaxed retention: log2 of this slot's weight r (0 for sinks and window keys),
    // and the partial sum of dS over the rows this thread sees, for dL/dr
    float bk2 = 0.f, dr_acc = 0.f;
    if (kColumn && a.bias != nullptr && key_row < nk) bk2 = __ldg(a.bias + col_base + kpos) * a.scale_log2;
    bool ok = true;
    for (int i = 0; i < n_rt && ok; ++i) {
      const int x = i & 1, st = i % kStagesK2;
      ok = mbar_wait(bar(K2_F + st), (i / kStagesK2) & 1, abort_flag, err, 418);   // row data
      if (ok) ok = mbar_wait(bar(K2_SF + x), (i >> 1) & 1, abort_flag, err, 419);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      const float* mf = reinterpret_cast<const float*>(sm + k2Meta) + st * 5 * kRowsK2;
      const int* mi = reinterpret_cast<const int*>(mf);
      // the rows of this tile that attend this key: one interval [r_a, r_b) of the
      // (token-major) rows; tokens past T never attend
      const int t0r = (rt0 + i) * TOK;
      const int r_end = min(kRowsK2, (a.T - t0r) * G);
      int r_a = 0, r_b = 0;
      if (key_row < nk) {
        if constexpr (!kColumn) {
          r_a = (kpos - t0r) * G;                          // tokens [kpos, kpos + w)
          r_b = (kpos + a.window - t0r) * G;
        } else if (kpos < a.sink) {
          r_a = (kpos + a.window - t0r) * G;               // tokens >= kpos + w
          r_b = kRowsK2;
        } else {
          // lo(t) <= i < hi(t) (and, lowest, hi(t) < death): hi and lo grow with t
          const int ii = kpos - a.sink, n = max(r_end, 0);
          r_a = first_above(mi + 4 * kRowsK2, n, ii);       // hi > i
          r_b = first_above(mi + 3 * kRowsK2, n, ii);       // lo > i
          if (lowest) r_b = min(r_b, first_above(mi + 4 * kRowsK2, n, kdeath - 1));
        }
        r_a = max(r_a, 0);
        r_b = min(r_b, r_end);
      }
      const uint32_t hb = (uint32_t)span64(r_a - 32 * half, r_b - 32 * half);   // this thread's 32 rows
      uint32_t rs[32], rp[32];
      tmem_ld32(lane_addr + (uint32_t)(x * 64 + 32 * half), rs);
      tmem_ld32(lane_addr + (uint32_t)(128 + x * 64 + 32 * half), rp);
      tmem_wait_ld();
      uint32_t pp[16], pd[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        float p2[2], d2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int rho = 32 * half + c + e;
          const bool on = (hb >> (c + e)) & 1u;
          const float p = on ? ex2(fmaf(__uint_as_float(rs[c + e]), a.scale_log2, bk2 - mf[rho])) : 0.f;
          p2[e] = p;
          d2[e] = on ? p * (__uint_as_float(rp[c + e]) - mf[kRowsK2 + rho]) : 0.f;
          if constexpr (kColumn) dr_acc += d2[e];
        }
        pp[c >> 1] = pk2(p2[0], p2[1]);
        pd[c >> 1] = pk2(d2[0], d2[1]);
      }
      // P^T, dS^T over the first 16 of this thread's 32 columns of S^T, dP^T
      tmem_st16(lane_addr + (uint32_t)(x * 64 + 32 * half), pp);
      tmem_st16(lane_addr + (uint32_t)(128 + x * 64 + 32 * half), pd);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(K2_PF + x));
    }
    ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(K2_DONE), 0, abort_flag, err, 420));
    if (ok) {
      tc_fence_after();
      // this thread: key row, dims [64 half, 64 half + 64) of dK and dV
      int pos = kpos;
      bool store = key_row < nk;
      if constexpr (kColumn) {
        if (store) {
          pos = kpos < a.sink ? kpos : __ldg(a.idx + crow + kpos - a.sink);
          store = pos < a.T;
        }
      }
      // dL/dr of a retained slot: sum of dS over its rows, over r (both halves add)
      if constexpr (kColumn) {
        if (store && a.dr != nullptr && kpos >= a.sink) atomicAdd(a.dr + crow + pos, dr_acc * ex2(-bk2));
      }
      const long long rowoff = (((long long)b * a.T + (store ? pos : 0)) * a.Hkv + h) * HD;
#pragma unroll 1
      for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
        uint32_t rk[32], rv[32];
        tmem_ld32(lane_addr + 384 + c0, rk);
        tmem_ld32(lane_addr + 256 + c0, rv);
        tmem_wait_ld();
        if (store) {
          float* dkr = a.dk + rowoff + c0;
          float* dvr = a.dv + rowoff + c0;
          if constexpr (kColumn) {
            // 16-byte vector atomics (rows are 512-byte aligned, c0 + e a multiple of 4)
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              atomicAdd(reinterpret_cast<float4*>(dkr + e),
                        make_float4(__uint_as_float(rk[e]) * a.scale, __uint_as_float(rk[e + 1]) * a.scale,
                                    __uint_as_float(rk[e + 2]) * a.scale, __uint_as_float(rk[e + 3]) * a.scale));
              atomicAdd(reinterpret_cast<float4*>(dvr + e),
                        make_float4(__uint_as_float(rv[e]), __uint_as_float(rv[e + 1]),
                                    __uint_as_float(rv[e + 2]), __uint_as_float(rv[e + 3])));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              *reinterpret_cast<float4*>(dkr + e) =
                  make_float4(__uint_as_float(rk[e]) * a.scale, __uint_as_float(rk[e + 1]) * a.scale,
                              __uint_as_float(rk[e + 2]) * a.scale, __uint_as_float(rk[e + 3]) * a.scale);
              *reinterpret_cast<float4*>(dvr + e) =
                  make_float4(__uint_as_float(rv[e]), __uint_as_float(rv[e + 1]),
                              __uint_as_float(rv[e + 2]), __uint_as_float(rv[e + 3]));
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                 : "memory");
}

}  // namespace bwdtc

bool attn_backward_dq_tc_supported(const lte_dims* d) {
  const int G = d->Hq / d->Hkv;
  return d->D == bwdtc::HD && (G == 1 || G == 2 || G == 4 || G == 8 || G == 16);
}

cudaError_t attn_backward_dkdv_tc(const bwd::Args& a, int B, DevError* err, cudaStream_t stream) {
  using namespace bwdtc;
  const int TOK = kRowsK2 / a.G;
  // tensor maps (contiguous bf16 rows of 128; 128-byte swizzle, 64-column boxes;
  // rows past a tensor's end read as zero)
  CUtensorMap mq, mdo, mk, mv, mkc, mvc;
  {
    const cuuint64_t dims[4] = {(cuuint64_t)HD, (cuuint64_t)a.Hq, (cuuint64_t)a.T, (cuuint64_t)B};
    const cuuint64_t st[3] = {(cuuint64_t)HD * 2, (cuuint64_t)a.Hq * HD * 2, (cuuint64_t)a.T * a.Hq * HD * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)a.G, (cuuint32_t)TOK, 1};
    if (!encode(&mq, a.q, 4, dims, st, box) || !encode(&mdo, a.dO, 4, dims, st, box))
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[4] = {(cuuint64_t)HD, (cuuint64_t)a.Hkv, (cuuint64_t)a.T, (cuuint64_t)B};
    const cuuint64_t st[3] = {(cuuint64_t)HD * 2, (cuuint64_t)a.Hkv * HD * 2,
                              (cuuint64_t)a.T * a.Hkv * HD * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)kKeysKV, 1};
    if (!encode(&mk, a.k, 4, dims, st, box) || !encode(&mv, a.v, 4, dims, st, box))
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t rows = (cuuint64_t)a.sink + a.T;
    const cuuint64_t dims[3] = {(cuuint64_t)HD, rows, (cuuint64_t)B * a.Hkv};
    const cuuint64_t st[2] = {(cuuint64_t)HD * 2, rows * HD * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kKeysKV, 1};
    if (!encode(&mkc, a.k_col, 3, dims, st, box) || !encode(&mvc, a.v_col, 3, dims, st, box))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_tc_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, k2Smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dkdv_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           k2Smem);
  if (e != cudaSuccess) return e;
  const int n_ktiles = (a.T + kKeysKV - 1) / kKeysKV;
  bwd_dkdv_tc_kernel<false><<<dim3(n_ktiles, a.Hkv, B), kThreadsK2, k2Smem, stream>>>(mq, mdo, mk, mv, a,
                                                                                     1, err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int n_ctiles = (a.sink + a.T + kKeysKV - 1) / kKeysKV;
  const int n_split = ((a.T + TOK - 1) / TOK + kSplitRowsK2 - 1) / kSplitRowsK2;
  const long long gx = (long long)n_ctiles * n_split;
  if (gx > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  bwd_dkdv_tc_kernel<true><<<dim3((unsigned)gx, a.Hkv, B), kThreadsK2, k2Smem, stream>>>(
      mq, mdo, mkc, mvc, a, n_split, err);
  return cudaGetLastError();
}

cudaError_t attn_backward_dq_tc(const bwd::Args& a, int B, DevError* err, cudaStream_t stream) {
  using namespace bwdtc;
  const int TOK = kRowsTc / a.G;
  // tensor maps (contiguous [B,T,H,128] bf16; 128-byte swizzle, 64-column boxes)
  CUtensorMap mq, mdo, mk, mv, mkc, mvc;
  {
    const cuuint64_t dims[4] = {(cuuint64_t)HD, (cuuint64_t)a.Hq, (cuuint64_t)a.T, (cuuint64_t)B};
    const cuuint64_t st[3] = {(cuuint64_t)HD * 2, (cuuint64_t)a.Hq * HD * 2, (cuuint64_t)a.T * a.Hq * HD * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)a.G, (cuuint32_t)TOK, 1};
    if (!encode(&mq, a.q, 4, dims, st, box) || !encode(&mdo, a.dO, 4, dims, st, box))
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[4] = {(cuuint64_t)HD, (cuuint64_t)a.Hkv, (cuuint64_t)a.T, (cuuint64_t)B};
    const cuuint64_t st[3] = {(cuuint64_t)HD * 2, (cuuint64_t)a.Hkv * HD * 2,
                              (cuuint64_t)a.T * a.Hkv * HD * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)kKeysTc, 1};
    if (!encode(&mk, a.k, 4, dims, st, box) || !encode(&mv, a.v, 4, dims, st, box))
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t rows = (cuuint64_t)a.sink + a.T;
    const cuuint64_t dims[3] = {(cuuint64_t)HD, rows, (cuuint64_t)B * a.Hkv};
    const cuuint64_t st[2] = {(cuuint64_t)HD * 2, rows * HD * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kKeysTc, 1};
    if (!encode(&mkc, a.k_col, 3, dims, st, box) || !encode(&mvc, a.v_col, 3, dims, st, box))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemP);
  if (e != cudaSuccess) return e;
  const int n_tiles = (a.T + TOK - 1) / TOK;
  bwd_dq_tc_kernel<<<dim3(n_tiles, a.Hkv, B), kThreadsP, kSmemP, stream>>>(mq, mdo, mk, mv, mkc, mvc,
                                                                          a, err);
  return cudaGetLastError();
}

}  // namespace lte
