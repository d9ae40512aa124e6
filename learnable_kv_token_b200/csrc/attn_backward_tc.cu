// Backward of the prefill sparse attention on 5th-generation tensor cores
// (tcgen05 + TMEM), head dim 128, bf16 operands, fp32 accumulation.
//
// "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention
// and Contextualized Learnable Token Eviction", Abstract (trained end to end)
// and Fig. 2 caption (right): the attended sets S_t, held fixed.  With P
// recomputed from the forward's lse and D_t = <dO_t, o_t>:
//   dS = P * (dO V^T - D_t),   dQ = scale dS K,   dV = P^T dO,   dK = scale dS^T Q.
//
// bwd_dq_tc_kernel: one CTA per 128 query rows (128/G tokens x the G heads of
// a KV head), over 64-key tiles of the rows' key ranges (sink slots and
// retained slots of the column segment, window band of k).
// bwd_dkdv_tc_kernel: persistent, one CTA per SM over work items of one
// 128-key tile (keys of k, or slots of the column segment) and a run of the
// 64-row query tiles that attend it.
// Both are warp-specialised: a TMA producer warp, a single-thread MMA issuer
// and eight row warps that form P and dS between the products; the roles are
// described above each kernel.  Every wait is bounded; on expiry the CTA
// records LTE_ERR_TIMEOUT, drains what it issued, frees its TMEM and leaves.
#include <math.h>

#include <type_traits>

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

// bits [a, b) of a 32-bit set (empty when b <= a), clipped to [0, 32)
__device__ __forceinline__ uint32_t span32(int a, int b) {
  a = a > 0 ? a : 0;
  b = b < 32 ? b : 32;
  if (b <= a) return 0u;
  return (0xffffffffu >> (32 - (b - a))) << a;
}
__device__ __forceinline__ uint32_t pk2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Roles (384 threads, one CTA per SM), per key tile j of the CTA's rows:
//   warp 0     TMA copies (one elected lane): K of tile j into a 7-stage ring
//              and V into a 4-stage ring (128-byte swizzled 64-column halves;
//              rows past the tensor read as zero) -- V is free once S(j), dP(j)
//              have completed, K only once dQ += dS(j) K(j) has;
//   warp 1     MMA issuer: S(j), dP(j) into TMEM buffer j % 2 (Q and dO are A
//              operands from TMEM), issued two tiles ahead of the rows, and
//              dQ += dS(j) K(j) once dS(j) is written: per rows' tile r it
//              issues dQ(r) and then S(r + 2), which reuses buffer r % 2 -- the
//              tensor core runs its products in issue order, so dQ(r) has read
//              dS(r) before S(r + 2) overwrites it;
//   warps 4-11 two threads per query row (warps 4-7 the first 32 keys of a
//              tile, 8-11 the last 32): Q and dO into TMEM at the start; P and
//              dS of tile j from TMEM buffer j % 2, dS written back as bf16
//              pairs over the first 16 of the 32 S columns each thread read
//              (no thread writes a column another still reads); at the end, dQ
//              out through a shared-memory stage, whole 512-byte rows per warp
//              store.
// TMEM: S[2] 0..127 (dS over them), dP[2] 128..255, dQ 256..383, Q 384..447,
// dO 448..511 (bf16 pairs).
constexpr int kThreadsP = 384;
constexpr int kStagesKP = 7, kStagesVP = 4;            // K and V rings
constexpr uint32_t kKR = 0;                             // K stage s at 16 KiB s
constexpr uint32_t kVR = kKR + kStagesKP * 16384;       // V stage s at 16 KiB s
constexpr uint32_t kOS = kVR + kStagesVP * 16384;       // o [128][128] bf16 (32 KiB), for D_t
constexpr uint32_t kDP = kOS + 32768;                   // [2][128] fp32 partial sums of D_t
constexpr uint32_t kBar2 = kDP + 2 * kRowsTc * 4;       // barriers
constexpr int kSmemP = kBar2 + 512;
constexpr uint32_t kColSP = 0, kColDPP = 128, kColDQP = 256, kColQP = 384, kColDOP = 448;
constexpr int kQStage = 3;                              // Q, dO arrive in K stages 3..6
constexpr uint32_t kQS = kKR + kQStage * 16384;         // Q [128][128] bf16 (32 KiB), then dO
static_assert(kQStage * 16384 + 65536 <= kStagesKP * 16384, "Q and dO fit the K ring's tail");
enum {
  P_QF = 0, P_QT = 1, P_KF = 2, P_KE = P_KF + kStagesKP, P_VF = P_KE + kStagesKP, P_VE = P_VF + kStagesVP,
  P_SF = P_VE + kStagesVP, P_DSF = P_SF + 2, P_DQ = P_DSF + 2,
  kNumBarsP = P_DQ + 1
};
static_assert(8 * kNumBarsP + 8 <= 512, "barriers fit");
static_assert(kSmemP <= 227 * 1024, "shared memory fits one CTA");
static_assert(kStagesKP * 16384 >= kRowsTc * HD * 4, "the K ring holds the dQ stage");

__global__ void __launch_bounds__(kThreadsP, 1)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_o,
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
    mbar_init(bar(P_QT), 256);
    for (int x = 0; x < kStagesKP; ++x) {
      mbar_init(bar(P_KF + x), 1);
      mbar_init(bar(P_KE + x), 1);
    }
    for (int x = 0; x < kStagesVP; ++x) {
      mbar_init(bar(P_VF + x), 1);
      mbar_init(bar(P_VE + x), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(P_SF + x), 1);
      mbar_init(bar(P_DSF + x), 256);
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
  int start0, count0, start1, count1, start2, count2;
  {
    int lo_f, n_first, lo_l, n_last;
    bwd::row_range(a, crow, t0, lo_f, n_first);
    bwd::row_range(a, crow, t_last, lo_l, n_last);
    const int lo_min = lowest ? 0 : lo_f;
    int nsink = t_last - a.window + 1;
    nsink = nsink < 0 ? 0 : (nsink > a.sink ? a.sink : nsink);
    nsink = nsink > a.T ? a.T : nsink;
    const int w_lo = t0 - a.window + 1 > 0 ? t0 - a.window + 1 : 0;
    start0 = 0; count0 = nsink;
    start1 = a.sink + lo_min; count1 = (a.cap > 0 && n_last > lo_min) ? n_last - lo_min : 0;
    start2 = w_lo; count2 = t_last - w_lo + 1;
  }
  const int n0 = (count0 + kKeysTc - 1) / kKeysTc, n1 = (count1 + kKeysTc - 1) / kKeysTc;
  const int total = n0 + n1 + (count2 + kKeysTc - 1) / kKeysTc;
  auto tile_of = [&](int j, int& rg, int& key0, int& nk) {   // (registers only)
    rg = j < n0 ? 0 : (j < n0 + n1 ? 1 : 2);
    const int it = j - (rg == 0 ? 0 : (rg == 1 ? n0 : n0 + n1));
    const int st_ = rg == 0 ? start0 : (rg == 1 ? start1 : start2);
    const int ct_ = rg == 0 ? count0 : (rg == 1 ? count1 : count2);
    key0 = st_ + it * kKeysTc;
    nk = min(kKeysTc, ct_ - it * kKeysTc);
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    bool ok = true;
    // Q and dO into K-ring stages kQStage .. (free until the rows have moved them
    // into TMEM)
    if (elect_one()) {
      mbar_expect_tx(bar(P_QF), 3 * kRowsTc * HD * 2);
      for (int hf = 0; hf < 2; ++hf) {
        tma_load_4d(sb + kQS + hf * (kRowsTc * 128), &tm_q, bar(P_QF), hf * 64, h * G, t0, b);
        tma_load_4d(sb + kQS + 32768u + hf * (kRowsTc * 128), &tm_do, bar(P_QF), hf * 64, h * G, t0, b);
        tma_load_4d(sb + kOS + hf * (kRowsTc * 128), &tm_o, bar(P_QF), hf * 64, h * G, t0, b);
      }
    }
    __syncwarp();
    int issued = 0;
    for (int j = 0; j < total && ok; ++j) {
      const int sk = j % kStagesKP, sv = j % kStagesVP;
      if (j >= kStagesKP && !(ok = wwait(bar(P_KE + sk), (j / kStagesKP - 1) & 1, abort_flag, err, 404))) break;
      if (j >= kQStage && j < kStagesKP && !(ok = wwait(bar(P_QT), 0, abort_flag, err, 414))) break;
      if (j >= kStagesVP && !(ok = wwait(bar(P_VE + sv), (j / kStagesVP - 1) & 1, abort_flag, err, 412))) break;
      int rg, key0, nk;
      tile_of(j, rg, key0, nk);
      if (elect_one()) {
        const uint32_t kd = sb + kKR + sk * 16384u, vd = sb + kVR + sv * 16384u;
        mbar_expect_tx(bar(P_KF + sk), kKeysTc * HD * 2);
        mbar_expect_tx(bar(P_VF + sv), kKeysTc * HD * 2);
        for (int hf = 0; hf < 2; ++hf) {
          if (rg == 2) {
            tma_load_4d(kd + hf * (kKeysTc * 128), &tm_k, bar(P_KF + sk), hf * 64, h, key0, b);
            tma_load_4d(vd + hf * (kKeysTc * 128), &tm_v, bar(P_VF + sv), hf * 64, h, key0, b);
          } else {
            tma_load_3d(kd + hf * (kKeysTc * 128), &tm_kc, bar(P_KF + sk), hf * 64, key0, u);
            tma_load_3d(vd + hf * (kKeysTc * 128), &tm_vc, bar(P_VF + sv), hf * 64, key0, u);
          }
        }
      }
      __syncwarp();
      issued = j + 1;
    }
    // every issued copy has landed before the CTA may exit
    mbar_drain(bar(P_QF), 0);
    for (int q = issued - kStagesKP > 0 ? issued - kStagesKP : 0; q < issued; ++q)
      mbar_drain(bar(P_KF + q % kStagesKP), (q / kStagesKP) & 1);
    for (int q = issued - kStagesVP > 0 ? issued - kStagesVP : 0; q < issued; ++q)
      mbar_drain(bar(P_VF + q % kStagesVP), (q / kStagesVP) & 1);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t id_s = idesc(kRowsTc, kKeysTc, false);     // S, dP: K-major A and B
    const uint32_t id_q = idesc(kRowsTc, HD, true);           // dQ: K as an N-contiguous B
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar(P_QT), 0, abort_flag, err, 405));
    auto issue_s = [&](int j) -> bool {                       // S(j), dP(j) into buffer j % 2
      const int x = j & 1, sk = j % kStagesKP, sv = j % kStagesVP;
      // (for j >= 2, dQ(j - 2) was issued just before: the rows have read S, dP
      // of tile j - 2, and the tensor core reads their dS before this overwrites it)
      bool w = mbar_wait(bar(P_KF + sk), (j / kStagesKP) & 1, abort_flag, err, 407);
      if (w) w = mbar_wait(bar(P_VF + sv), (j / kStagesVP) & 1, abort_flag, err, 413);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint64_t dk = sdesc(sb + kKR + sk * 16384u, 16, 1024);
        const uint64_t dv = sdesc(sb + kVR + sv * 16384u, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
          const uint32_t ob = ((ks >> 2) * (kKeysTc * 128) + (ks & 3) * 32) >> 4;
          mma_f16_ts(tmem + kColSP + x * 64, tmem + kColQP + 8 * ks, dk + ob, id_s, ks > 0 ? 1u : 0u);
          mma_f16_ts(tmem + kColDPP + x * 64, tmem + kColDOP + 8 * ks, dv + ob, id_s, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar(P_SF + x));
        mma_commit(bar(P_VE + sv));                           // V of tile j is free
      }
      __syncwarp();
      return true;
    };
    auto issue_dq = [&](int jj) -> bool {                     // dQ += dS(jj) K(jj)
      const int x = jj & 1, sk = jj % kStagesKP;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(P_DSF + x), (jj >> 1) & 1, abort_flag, err, 406)))
        return false;
      tc_fence_after();
      if (elect_one()) {
        const uint64_t dkb = sdesc(sb + kKR + sk * 16384u, kKeysTc * 128, 1024);
#pragma unroll
        for (int ks = 0; ks < kKeysTc / 16; ++ks) {
          // keys 16 ks ..: the packed dS a row's thread (ks >> 1) wrote over the first
          // 16 of its 32 columns of S buffer x
          const uint32_t pc = (uint32_t)(x * 64 + 32 * (ks >> 1) + 8 * (ks & 1));
          mma_f16_ts(tmem + kColDQP, tmem + kColSP + pc, dkb + ((ks * 2048) >> 4), id_q,
                     (jj > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(bar(P_KE + sk));                           // K of tile jj is free
      }
      __syncwarp();
      return true;
    };
    if (ok && total > 0) ok = issue_s(0);
    if (ok && total > 1) ok = issue_s(1);
    for (int r = 0; r < total && ok; ++r) {
      ok = issue_dq(r);
      if (ok && r + 2 < total) ok = issue_s(r + 2);
    }
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
    // Q and dO of this row, dims [64 kh, 64 kh + 64), from their 128-byte swizzled
    // halves in shared memory (zeros past T, as the copy fills them) into TMEM;
    // with o, this half's part of D_t = <dO_t, o_t>
    float* dpart = reinterpret_cast<float*>(sm + kDP);
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar(P_QF), 0, abort_flag, err, 415));
    {
      float dsum = 0.f;
      if (ok) {
        uint32_t rq[32], rd[32];
        const uint8_t* qrow = sm + kQS + kh * (kRowsTc * 128) + row * 128;
        const uint8_t* orow = sm + kOS + kh * (kRowsTc * 128) + row * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int off = (c ^ (row & 7)) << 4;
          const uint4 vq = *reinterpret_cast<const uint4*>(qrow + off);
          const uint4 vd = *reinterpret_cast<const uint4*>(qrow + 32768 + off);
          const uint4 vo = *reinterpret_cast<const uint4*>(orow + off);
          rq[4 * c] = vq.x, rq[4 * c + 1] = vq.y, rq[4 * c + 2] = vq.z, rq[4 * c + 3] = vq.w;
          rd[4 * c] = vd.x, rd[4 * c + 1] = vd.y, rd[4 * c + 2] = vd.z, rd[4 * c + 3] = vd.w;
          const uint32_t ow[4] = {vo.x, vo.y, vo.z, vo.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 xo = *reinterpret_cast<const __nv_bfloat162*>(&ow[e]);
            const __nv_bfloat162 xd = *reinterpret_cast<const __nv_bfloat162*>(&rd[4 * c + e]);
            dsum = fmaf(__low2float(xo), __low2float(xd), dsum);
            dsum = fmaf(__high2float(xo), __high2float(xd), dsum);
          }
        }
        tmem_st32(lane_addr + kColQP + 32 * kh, rq);
        tmem_st32(lane_addr + kColDOP + 32 * kh, rd);
        tmem_wait_st();
      }
      dpart[kh * kRowsTc + row] = dsum;
    }
    tc_fence_before();
    mbar_arrive(bar(P_QT));                            // (also on a failed wait: never blocks the others)
    bar_sync(1, 256);                                  // both halves of every D_t are in dpart
    int lo_r, hi_r;
    bwd::row_range(a, crow, tt, lo_r, hi_r);
    if (lowest) lo_r = 0;
    // D_t for this row (written out once for the dK/dV passes) and the row's lse
    float lse2 = 0.f, dl = 0.f;
    if (tt < a.T) {
      const long long li = ((long long)b * a.Hq + h * G + gq) * a.T + tt;
      lse2 = a.lse[li] * 1.4426950408889634f;
      dl = dpart[row] + dpart[kRowsTc + row];
      if (kh == 0) a.delta[li] = dl;
    }
    for (int j = 0; j < total && ok; ++j) {
      const int x = j & 1;
      int rg, key0, nk;
      tile_of(j, rg, key0, nk);
      // this row's keys among this thread's 32 (keys kb .. kb + 31 of the tile's
      // positions or slots): at most two intervals (sink slots, retained slots
      // [lo, hi)) or one (window band)
      const int kb = key0 + 32 * kh, nkh = nk - 32 * kh;
      uint32_t hb = 0u;
      if (tt < a.T) {
        if (rg == 2) {
          hb = span32(tt - a.window + 1 - kb, min(nkh, tt - kb + 1));
        } else {
          const int sink_end = min(a.sink, tt - a.window + 1);
          uint32_t ret = span32(a.sink + lo_r - kb, min(nkh, a.sink + hi_r - kb));
          if (lowest && ret != 0u) {                   // lifetimes: held at count hi_r
#pragma unroll 4
            for (int kk = 0; kk < 32; ++kk)
              if (((ret >> kk) & 1u) && __ldg(a.death + crow + kb + kk - a.sink) <= hi_r)
                ret &= ~(1u << kk);
          }
          hb = span32(-kb, min(nkh, sink_end - kb)) | ret;
        }
      }
      const float* brow = (a.bias != nullptr && rg != 2) ? a.bias + col_base + key0 + 32 * kh : nullptr;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(P_SF + x), (j >> 1) & 1, abort_flag, err, 409))))
        break;
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
        // dS = P (dP - D); a row that attends all 32 keys (the common case) takes
        // the unmasked form
        auto form = [&](auto all_on) {
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            float ds2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              float p = ex2(fmaf(__uint_as_float(rs[c + e]), a.scale_log2, -lse2));
              if constexpr (!decltype(all_on)::value) p = ((hb >> (c + e)) & 1u) ? p : 0.f;
              ds2[e] = p * (__uint_as_float(rp[c + e]) - dl);
            }
            pkd[c >> 1] = pk2(ds2[0], ds2[1]);
          }
        };
        if (hb == 0xffffffffu) form(std::true_type{});
        else form(std::false_type{});
      }
      // dS of keys 32 kh .. as bf16 pairs over the first 16 of the 32 S columns this
      // thread has read: the A operand of dQ += dS K
      tmem_st16(lane_addr + kColSP + x * 64 + 32 * kh, pkd);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(P_DSF + x));
    }
    // dQ out.  Once every product has completed (and so every K, V copy has
    // landed and been read), each thread stages its row's 64 columns (x scale) in
    // the K ring, 16-byte chunks XOR-swizzled by row, then each warp writes
    // whole 512-byte rows.  The eight row warps go on together or stop together
    // (named barrier 1).
    ok = ok && mbar_wait(bar(P_DQ), 0, abort_flag, err, 411);
    ok = bar_and(1, 256, __all_sync(0xffffffffu, ok));
    if (ok) {
      tc_fence_after();
      uint8_t* stage = sm + kKR;                         // [128][128] fp32
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
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const int ch = (c0 + e) >> 2;                  // 16-byte chunk of the 512-byte row
          *reinterpret_cast<float4*>(stage + row * 512 + ((ch ^ (row & 31)) << 4)) =
              make_float4(__uint_as_float(r[e]) * a.scale, __uint_as_float(r[e + 1]) * a.scale,
                          __uint_as_float(r[e + 2]) * a.scale, __uint_as_float(r[e + 3]) * a.scale);
        }
      }
      bar_sync(1, 256);
      const int lane = tid & 31, w8 = warp - 4;
#pragma unroll 4
      for (int rr = w8; rr < kRowsTc; rr += 8) {
        const int t_r = t0 + rr / G;
        if (t_r < a.T) {
          const float4 v = *reinterpret_cast<const float4*>(stage + rr * 512 + ((lane ^ (rr & 31)) << 4));
          float* out = a.dq + (((long long)b * a.T + t_r) * a.Hq + h * G + rr % G) * HD;
          *reinterpret_cast<float4*>(out + 4 * lane) = v;
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
// Persistent: one CTA per SM takes work items in a static stride.  An item is
// a 128-key tile and a run of the query-row tiles that attend it: for the
// window part (kColumn = false) the keys of k, item = (b, h, tile), all rows
// t in [j, j + w); for the column part (kColumn = true) slots of the column
// segment, items from the list bwd_col_items_kernel writes (a slot's rows are
// split into runs of about kSplitRowsK2 row tiles, so several CTAs share a
// busy tile and add into dK, dV with atomics).  Keys are the MMA rows; the
// attending query rows come in tiles of 64 (64/G tokens x the G heads), and
// per row tile:
//   S^T = K Q^T, dP^T = V dO^T        (M128 N64 K128) into TMEM buffer g % 2
//   P^T, dS^T = P^T (dP^T - D)         (two threads per key row, 32 rows each),
//                                      as bf16 over the columns of S^T and dP^T
//                                      each thread read
//   dV += P^T dO, dK += dS^T Q         (M128 N128 K64; P^T, dS^T read from TMEM)
// The tensor core runs its products in issue order.  The MMA thread issues
// S^T two row tiles ahead of the rows (across items: K and V of the next item
// arrive once the current item's last S^T has completed) and, per row tile g,
// dV and dK of g once its P^T and dS^T are written, then S^T of g + 2 into the
// same buffer -- so S^T of a tile never waits behind a product that waits for
// the rows, and the rows never wait for S^T.
// Roles (384 threads):
//   warp 0     TMA producer (one elected lane): K and V of each item, once the
//              item before has issued its last S^T and that has completed; per
//              row tile, Q and dO into a 4-stage ring, then the rows' lse and D
//              and the tokens' retained range, written by the warp's lanes
//              while the copies fly;
//   warp 1     MMA issuer, as above;
//   warps 4-11 two threads per key row (warps 4-7 rows 0-31 of a tile, 8-11
//              rows 32-63): P^T and dS^T, each written over the first 16 of the
//              32 columns of S^T (dP^T) the thread read, so no thread writes a
//              column another still reads; at the end of an item, dK and dV out
//              through a shared-memory stage in 32-column chunks, so that each
//              warp store (or add) covers four whole 128-byte rows, while the
//              tensor core already computes the next item's first S^T.
// TMEM: S^T of buffer x at 64 x (P^T over it), dP^T at 128 + 64 x (dS^T over
// it), dV 256..383, dK 384..511.  Barrier phases run on a row-tile counter that
// continues across items (ring stages, S^T buffers) or on the item counter (K
// and V, items' completion).
constexpr int kKeysKV = 128;
constexpr int kRowsK2 = 64;                       // attending query rows per tile
constexpr int kStagesK2 = 4;
constexpr int kThreadsK2 = 384;
constexpr int kSplitRowsK2 = 64;                  // row tiles per column item, at most
constexpr uint32_t k2K = 0, k2V = 32768;          // [128][128] bf16 each: halves of 16 KiB
constexpr uint32_t k2QD = 65536;                  // stage s: Q at + 32 KiB s, dO at + 16 KiB
constexpr uint32_t k2Meta = k2QD + kStagesK2 * 32768;            // stage s: [5][64] words
constexpr uint32_t k2Stage = k2Meta + kStagesK2 * 5 * kRowsK2 * 4;   // [128][32] fp32, swizzled
constexpr uint32_t k2Pos = k2Stage + kKeysKV * 128;                  // [128] output row per key
constexpr uint32_t k2Bar = k2Pos + kKeysKV * 4;
constexpr int k2Smem = k2Bar + 256;
constexpr uint32_t k2ColS = 0, k2ColDP = 128, k2ColDV = 256, k2ColDK = 384;
enum {
  K2_KVF = 0, K2_KVE = 1, K2_F = 2, K2_E = K2_F + kStagesK2, K2_SF = K2_E + kStagesK2, K2_PF = K2_SF + 2,
  K2_DONE = K2_PF + 2, kNumBarsK2 = K2_DONE + 1
};
static_assert(8 * kNumBarsK2 + 16 <= 256, "barriers and flags fit");
static_assert(k2Smem <= 227 * 1024, "shared memory fits one CTA");

// One work item: KV unit u = b Hkv + h, key tile, first row tile, row tiles.
struct K2Item {
  int u, tile, rt0, n_rt;
};

// Warp-wide: first m in [l, r) with pred(m) true for a predicate that is false
// then true over [l, r) (r if none); every lane returns it.  Rounds of 32 probes.
template <class Pred>
__device__ __forceinline__ int warp_first_true(int l, int r, int lane, Pred pred) {
  while (r - l > 32) {
    const int step = (r - l + 31) / 32;
    const int p = l + lane * step;
    const unsigned hit = __ballot_sync(0xffffffffu, p < r && pred(p));
    const unsigned probed = __ballot_sync(0xffffffffu, p < r);
    if (hit == 0u) {
      l = l + (31 - __clz(probed)) * step + 1;           // past the last probe
    } else {
      const int f = __ffs(hit) - 1;
      if (f == 0) return l;
      r = l + f * step;                                   // true there
      l = l + (f - 1) * step + 1;
    }
  }
  const int p = l + lane;
  const unsigned hit = __ballot_sync(0xffffffffu, p < r && pred(p));
  return hit ? l + __ffs(hit) - 1 : r;
}

// The column part's work list: one CTA per KV unit, one warp per slot tile
// (32 tiles per round); the query tokens [lo_t, hi_t] that attend some slot of
// the tile (the same bounds the row masks use: a sink slot j is attended by
// rows t >= j + w, a retained slot i by the rows whose retained count n_t,
// nondecreasing in t, holds it), cut into runs of at most kSplitRowsK2 row
// tiles of near-equal length.  Each round's items are written in tile order
// at a block reserved with one atomic, so a unit's items sit together: CTAs
// that take neighbouring items work on the same unit's Q and dO, which then
// stay in L2.
constexpr int kColItemsThreads = 1024;
__global__ void __launch_bounds__(kColItemsThreads)
bwd_col_items_kernel(const bwd::Args a, int n_ctiles, K2Item* items, int* n_items) {
  __shared__ int rt0_sh[32], n_sh[32], runs_sh[32], off_sh[33];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int u = blockIdx.x;
  const long long crow = (long long)u * a.T;
  const int nret = __ldg(a.nret + u);
  const int TOK = kRowsK2 / a.G;
  for (int base_tile = 0; base_tile < n_ctiles; base_tile += 32) {
    const int tile = base_tile + wid;
    const int k0 = tile * kKeysKV;
    const int nk = tile < n_ctiles ? min(kKeysKV, a.sink + nret - k0) : 0;
    int lo_t = a.T, hi_t = -1;
    if (nk > 0) {
      const int s_end = min(min(a.sink, k0 + nk), a.T);
      if (k0 < s_end) {
        lo_t = k0 + a.window;
        hi_t = a.T - 1;
      }
      const int i0 = max(k0, a.sink) - a.sink, i1 = k0 + nk - a.sink;
      if (i1 > i0 && a.cap > 0 && (a.cap_policy != LTE_CAP_FIRST || i0 < a.cap) && a.window < a.T) {
        auto cnt = [&](int t) { return __ldg(a.cnt + crow + t - a.window); };   // rows t >= w
        const int l = warp_first_true(a.window, a.T, lane, [&](int m) { return cnt(m) > i0; });
        if (l < a.T) {
          long long bound;                                 // rows need cnt < bound
          if (a.cap_policy == LTE_CAP_RECENT) bound = (long long)i1 + a.cap;
          else if (a.cap_policy == LTE_CAP_FIRST) bound = 1ll << 40;
          else {
            int md = 0;
            for (int i = i0 + lane; i < i1; i += 32) md = max(md, __ldg(a.death + crow + i));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) md = max(md, __shfl_xor_sync(0xffffffffu, md, o));
            bound = md;
          }
          const int l2 = warp_first_true(l, a.T, lane, [&](int m) { return (long long)cnt(m) >= bound; });
          if (l2 > l) {
            lo_t = min(lo_t, l);
            hi_t = max(hi_t, l2 - 1);
          }
        }
      }
    }
    if (lane == 0) {
      int r0 = 0, n = 0, runs = 0;
      if (lo_t <= hi_t) {
        r0 = lo_t / TOK;
        n = hi_t / TOK - r0 + 1;
        runs = (n + kSplitRowsK2 - 1) / kSplitRowsK2;
      }
      rt0_sh[wid] = r0, n_sh[wid] = n, runs_sh[wid] = runs;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int acc = 0;
      for (int w = 0; w < 32; ++w) off_sh[w] = acc, acc += runs_sh[w];
      off_sh[32] = acc > 0 ? atomicAdd(n_items, acc) : 0;
    }
    __syncthreads();
    if (lane == 0 && runs_sh[wid] > 0) {
      const int n = n_sh[wid], runs = runs_sh[wid], len = (n + runs - 1) / runs;
      K2Item* dst = items + off_sh[32] + off_sh[wid];
      for (int c = 0; c < runs; ++c) dst[c] = K2Item{u, tile, rt0_sh[wid] + c * len, min(len, n - c * len)};
    }
    __syncthreads();                                       // the round's arrays may be reused
  }
}

template <bool kColumn>
__global__ void __launch_bounds__(kThreadsK2, 1)
bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const bwd::Args a, const K2Item* items,
                   const int* n_items_p, int n_items_win, DevError* err) {
  extern __shared__ __align__(1024) uint8_t sm[];
  const uint32_t sb = sa(sm);
  if ((sb & 1023u) != 0) {
    if (threadIdx.x == 0) record_error(err, LTE_ERR_DEVICE, 413);
    return;
  }
  const int n_items = kColumn ? __ldg(n_items_p) : n_items_win;
  if ((int)blockIdx.x >= n_items) return;              // no work (uniform)
  auto bar = [&](int i) { return sb + k2Bar + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + k2Bar + 8 * kNumBarsK2);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + k2Bar + 8 * kNumBarsK2 + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G, TOK = kRowsK2 / G;
  const bool lowest = a.death != nullptr;
  const int n_ktiles = (a.T + kKeysKV - 1) / kKeysKV;
  // item `it` -> KV unit, key tile, its row tiles [rt0, rt0 + n_rt) and keys
  auto item_at = [&](int it) {
    K2Item w;
    if constexpr (kColumn) {
      w = items[it];
    } else {
      w.tile = it % n_ktiles;
      w.u = it / n_ktiles;
      const int k0 = w.tile * kKeysKV, nk = min(kKeysKV, a.T - k0);
      w.rt0 = k0 / TOK;                                  // rows t in [k0, k0 + nk - 1 + w - 1]
      w.n_rt = min(a.T - 1, k0 + nk - 1 + a.window - 1) / TOK - w.rt0 + 1;
    }
    return w;
  };
  auto keys_of = [&](const K2Item& w) {
    const int k0 = w.tile * kKeysKV;
    return kColumn ? min(kKeysKV, a.sink + __ldg(a.nret + w.u) - k0) : min(kKeysKV, a.T - k0);
  };

  if (tid == 0) {
    mbar_init(bar(K2_KVF), 1);
    mbar_init(bar(K2_KVE), 1);
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
    int g = 0, k = 0;                                      // row tiles, items issued
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++k) {
      const K2Item w = item_at(it);
      const int h = w.u % a.Hkv, b = w.u / a.Hkv, k0 = w.tile * kKeysKV;
      const long long crow = (long long)w.u * a.T;
      // K and V: the previous item's last S^T, dP^T have completed
      if (k >= 1 && !(ok = wwait(bar(K2_KVE), (k - 1) & 1, abort_flag, err, 424))) break;
      if (elect_one()) {
        mbar_expect_tx(bar(K2_KVF), 2 * kKeysKV * HD * 2);
        for (int hf = 0; hf < 2; ++hf) {
          if constexpr (kColumn) {
            tma_load_3d(sb + k2K + hf * 16384u, &tm_k, bar(K2_KVF), hf * 64, k0, w.u);
            tma_load_3d(sb + k2V + hf * 16384u, &tm_v, bar(K2_KVF), hf * 64, k0, w.u);
          } else {
            tma_load_4d(sb + k2K + hf * 16384u, &tm_k, bar(K2_KVF), hf * 64, h, k0, b);
            tma_load_4d(sb + k2V + hf * 16384u, &tm_v, bar(K2_KVF), hf * 64, h, k0, b);
          }
        }
      }
      __syncwarp();
      for (int i = 0; i < w.n_rt; ++i, ++g) {
        const int st = g % kStagesK2, use = g / kStagesK2;
        if (use >= 1 && !(ok = wwait(bar(K2_E + st), (use - 1) & 1, abort_flag, err, 414))) break;
        const int t0r = (w.rt0 + i) * TOK;
        // the copies first (the phase also waits for the arrive below) ...
        if (elect_one()) {
          const uint32_t qs = sb + k2QD + st * 32768u;
          mbar_add_tx(bar(K2_F + st), 2 * kRowsK2 * HD * 2);
          for (int hf = 0; hf < 2; ++hf) {
            tma_load_4d(qs + hf * 8192u, &tm_q, bar(K2_F + st), hf * 64, h * G, t0r, b);
            tma_load_4d(qs + 16384u + hf * 8192u, &tm_do, bar(K2_F + st), hf * 64, h * G, t0r, b);
          }
        }
        // ... then the rows' data: lse (log2) and D per row; the retained range
        // [lo, hi) per token (j < 64/G), INT_MAX for tokens past T
        float* mf = reinterpret_cast<float*>(sm + k2Meta) + st * 5 * kRowsK2;
        int* mi = reinterpret_cast<int*>(mf);
        float l2[2], dd[2];
        int cv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int r = lane + 32 * e, tt = t0r + r / G, gg = r % G, tj = t0r + r;
          l2[e] = 0.f, dd[e] = 0.f, cv[e] = 0;
          if (tt < a.T) {
            const long long li = ((long long)b * a.Hq + h * G + gg) * a.T + tt;
            l2[e] = __ldg(a.lse + li);
            dd[e] = __ldg(a.delta + li);
          }
          if (kColumn && r < TOK && tj < a.T && tj >= a.window) cv[e] = __ldg(a.cnt + crow + tj - a.window);
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int r = lane + 32 * e, tj = t0r + r;
          mf[r] = l2[e] * 1.4426950408889634f;
          mf[kRowsK2 + r] = dd[e];
          if (kColumn && r < TOK) {
            int hi = INT_MAX, lo = INT_MAX;
            if (tj < a.T) {
              hi = tj >= a.window ? held_retained(cv[e], a.cap, a.cap_policy) : 0;
              lo = (!lowest && a.cap_policy == LTE_CAP_RECENT && hi - a.cap > 0) ? hi - a.cap : 0;
            }
            mi[3 * kRowsK2 + r] = lo;
            mi[4 * kRowsK2 + r] = hi;
          }
        }
        __syncwarp();
        if (elect_one()) mbar_arrive(bar(K2_F + st));
        __syncwarp();
      }
    }
    // every issued copy has landed before the CTA may exit
    if (k >= 1) mbar_drain(bar(K2_KVF), (k - 1) & 1);
    for (int q = g - kStagesK2 > 0 ? g - kStagesK2 : 0; q < g; ++q)
      mbar_drain(bar(K2_F + q % kStagesK2), (q / kStagesK2) & 1);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t id_s = idesc(kKeysKV, kRowsK2, false);    // S^T, dP^T: K-major A and B
    const uint32_t id_o = idesc(kKeysKV, HD, true);          // dV, dK: dO, Q as N-contiguous B
    bool ok = true;
    auto issue_dvdk = [&](int gg, bool first) -> bool {      // dV, dK of row tile gg
      const int st = gg % kStagesK2, x = gg & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(K2_PF + x), (gg >> 1) & 1, abort_flag, err, 416))) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t qs = sb + k2QD + st * 32768u;
        const uint64_t qb = sdesc(qs, kRowsK2 * 128, 1024), dob = sdesc(qs + 16384u, kRowsK2 * 128, 1024);
#pragma unroll
        for (int ks = 0; ks < kRowsK2 / 16; ++ks) {
          // rows 16 ks ..: packed by the thread of row half ks >> 1 over the first 16
          // of its 32 columns of buffer x
          const uint32_t pc = (uint32_t)(x * 64 + 32 * (ks >> 1) + 8 * (ks & 1));
          const uint32_t acc = (!first || ks > 0) ? 1u : 0u;
          mma_f16_ts(tmem + k2ColDV, tmem + k2ColS + pc, dob + ((ks * 2048) >> 4), id_o, acc);
          mma_f16_ts(tmem + k2ColDK, tmem + k2ColDP + pc, qb + ((ks * 2048) >> 4), id_o, acc);
        }
        mma_commit(bar(K2_E + st));                          // the row tile's stage is free
      }
      __syncwarp();
      return true;
    };
    // S^T stream: a cursor over (item, row tile) that runs two tiles ahead
    int s_item = blockIdx.x, s_k = 0, s_i = 0, s_n = item_at(s_item).n_rt, gs = 0;
    auto issue_next_s = [&]() -> bool {
      if (s_item >= n_items) return true;                     // nothing left to start
      const int st = gs % kStagesK2, x = gs & 1;
      // (for gs >= 2, dV and dK of gs - 2 were issued just before: they read
      // P^T, dS^T from this buffer before S^T of gs overwrites it)
      bool w = true;
      if (s_i == 0) w = mbar_wait(bar(K2_KVF), s_k & 1, abort_flag, err, 415);   // K, V of the item
      if (w) w = mbar_wait(bar(K2_F + st), (gs / kStagesK2) & 1, abort_flag, err, 417);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t qs = sb + k2QD + st * 32768u;
        const uint64_t dk = sdesc(sb + k2K, 16, 1024), dv = sdesc(sb + k2V, 16, 1024);
        const uint64_t dq = sdesc(qs, 16, 1024), ddo = sdesc(qs + 16384u, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
          const uint32_t oa = ((ks >> 2) * (kKeysKV * 128) + (ks & 3) * 32) >> 4;
          const uint32_t ob = ((ks >> 2) * (kRowsK2 * 128) + (ks & 3) * 32) >> 4;
          mma_f16(tmem + k2ColS + x * 64, dk + oa, dq + ob, id_s, ks > 0 ? 1u : 0u);
          mma_f16(tmem + k2ColDP + x * 64, dv + oa, ddo + ob, id_s, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar(K2_SF + x));
        if (s_i == s_n - 1) mma_commit(bar(K2_KVE));         // K, V of the item no longer read
      }
      __syncwarp();
      ++gs;
      if (++s_i == s_n) {
        s_i = 0;
        ++s_k;
        s_item += gridDim.x;
        if (s_item < n_items) s_n = item_at(s_item).n_rt;
      }
      return true;
    };
    ok = issue_next_s();
    if (ok) ok = issue_next_s();
    int g = 0, k = 0;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++k) {
      const int n_rt = item_at(it).n_rt;
      bool done = false;
      for (int i = 0; i < n_rt && ok; ++i, ++g) {
        ok = issue_dvdk(g, i == 0);
        if (ok && i == n_rt - 1) {
          // every product of the item has completed (before S^T of the next
          // item's tiles that follow in the queue)
          if (elect_one()) mma_commit(bar(K2_DONE));
          __syncwarp();
          done = true;
        }
        if (ok) ok = issue_next_s();
      }
      if (!done) {
        if (elect_one()) mma_commit(bar(K2_DONE));
        __syncwarp();
      }
    }
    if (k >= 1) mbar_drain(bar(K2_DONE), (k - 1) & 1);
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- key rows (warps 4-11)
    const int quad = warp & 3, half = (warp - 4) >> 2;     // TMEM lane quadrant, row half
    const int key_row = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    bool ok = true;
    int g = 0, k = 0;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++k) {
      const K2Item w = item_at(it);
      const int h = w.u % a.Hkv, b = w.u / a.Hkv, k0 = w.tile * kKeysKV, nk = keys_of(w);
      const long long crow = (long long)w.u * a.T;
      const long long col_base = (long long)w.u * (a.sink + a.T);
      const int kpos = k0 + key_row;                       // position (window) or slot (column)
      int kdeath = 0;
      if (kColumn && lowest && kpos >= a.sink && key_row < nk) kdeath = __ldg(a.death + crow + kpos - a.sink);
      // relaxed retention: log2 of this slot's weight r (0 for sinks and window keys),
      // and the partial sum of dS over the rows this thread sees, for dL/dr
      float bk2 = 0.f, dr_acc = 0.f;
      if (kColumn && a.bias != nullptr && key_row < nk) bk2 = __ldg(a.bias + col_base + kpos) * a.scale_log2;
      for (int i = 0; i < w.n_rt; ++i, ++g) {
        const int st = g % kStagesK2;
        // the row data first: the rows' range is found while S^T is computed
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(K2_F + st), (g / kStagesK2) & 1, abort_flag, err, 418))))
          break;
        const float* mf = reinterpret_cast<const float*>(sm + k2Meta) + st * 5 * kRowsK2;
        const int* mi = reinterpret_cast<const int*>(mf);
        // the rows of this tile that attend this key: one interval [r_a, r_b) of the
        // (token-major) rows; tokens past T never attend
        const int t0r = (w.rt0 + i) * TOK;
        const int r_end = min(kRowsK2, (a.T - t0r) * G);
        int r_a = 0, r_b = 0;
        if (key_row < nk) {
          if constexpr (!kColumn) {
            r_a = (kpos - t0r) * G;                        // tokens [kpos, kpos + w)
            r_b = (kpos + a.window - t0r) * G;
          } else if (kpos < a.sink) {
            r_a = (kpos + a.window - t0r) * G;             // tokens >= kpos + w
            r_b = kRowsK2;
          } else {
            // lo(t) <= i < hi(t) (and, lowest, hi(t) < death): hi and lo grow with t
            // (INT_MAX past T), so the first token above a bound is the count of
            // tokens at or below it -- counted over broadcast reads
            const int ii = kpos - a.sink, hd = lowest ? kdeath - 1 : INT_MAX - 1;
            int ca = 0, cb = 0, cd = 0;
            for (int j = 0; j < TOK; j += 4) {
              const int4 hv = *reinterpret_cast<const int4*>(mi + 4 * kRowsK2 + j);
              const int4 lv = *reinterpret_cast<const int4*>(mi + 3 * kRowsK2 + j);
              ca += (hv.x <= ii) + (hv.y <= ii) + (hv.z <= ii) + (hv.w <= ii);
              cb += (lv.x <= ii) + (lv.y <= ii) + (lv.z <= ii) + (lv.w <= ii);
              cd += (hv.x <= hd) + (hv.y <= hd) + (hv.z <= hd) + (hv.w <= hd);
            }
            r_a = G * ca;                                  // first row with hi > i
            r_b = G * min(cb, cd);                         // first row with lo > i (or hi >= death)
          }
          r_a = max(r_a, 0);
          r_b = min(r_b, r_end);
        }
        const uint32_t hb = span32(r_a - 32 * half, r_b - 32 * half);   // this thread's 32 rows
        const int x = g & 1;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(bar(K2_SF + x), (g >> 1) & 1, abort_flag, err, 419))))
          break;
        tc_fence_after();
        uint32_t rs[32], rp[32];
        tmem_ld32(lane_addr + k2ColS + x * 64 + 32 * half, rs);
        tmem_ld32(lane_addr + k2ColDP + x * 64 + 32 * half, rp);
        tmem_wait_ld();
        const float4* ml = reinterpret_cast<const float4*>(mf + 32 * half);
        const float4* md = reinterpret_cast<const float4*>(mf + kRowsK2 + 32 * half);
        uint32_t pp[16], pd[16];
        // P^T, dS^T; a key that all 32 rows attend (the common case) takes the
        // unmasked form
        auto form = [&](auto all_on) {
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const float4 l4 = ml[c4], d4 = md[c4];
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv4[4] = {d4.x, d4.y, d4.z, d4.w};
            float p4[4], q4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 4 * c4 + e;
              float p = ex2(fmaf(__uint_as_float(rs[c]), a.scale_log2, bk2 - lv[e]));
              float q = p * (__uint_as_float(rp[c]) - dv4[e]);
              if constexpr (!decltype(all_on)::value) {
                const bool on = (hb >> c) & 1u;
                p = on ? p : 0.f;
                q = on ? q : 0.f;
              }
              p4[e] = p;
              q4[e] = q;
              if constexpr (kColumn) dr_acc += q;
            }
            pp[2 * c4] = pk2(p4[0], p4[1]);
            pp[2 * c4 + 1] = pk2(p4[2], p4[3]);
            pd[2 * c4] = pk2(q4[0], q4[1]);
            pd[2 * c4 + 1] = pk2(q4[2], q4[3]);
          }
        };
        if (hb == 0xffffffffu) form(std::true_type{});
        else form(std::false_type{});
        // rows 32 half .. + 31 of P^T, dS^T over the first 16 of the 32 columns of
        // S^T, dP^T this thread read
        tmem_st16(lane_addr + k2ColS + (uint32_t)(64 * x + 32 * half), pp);
        tmem_st16(lane_addr + k2ColDP + (uint32_t)(64 * x + 32 * half), pd);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(K2_PF + x));
      }
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(K2_DONE), k & 1, abort_flag, err, 420));
      // the eight row warps go on together or stop together (the stage below
      // synchronises them with a named barrier)
      if (!(ok = bar_and(1, 256, ok))) break;
      tc_fence_after();
      // this thread's key row: output row (-1: none), and dL/dr of a retained slot
      // (sum of dS over its rows, over r; both halves add)
      int pos = kpos;
      bool store = key_row < nk;
      if constexpr (kColumn) {
        if (store) {
          pos = kpos < a.sink ? kpos : __ldg(a.idx + crow + kpos - a.sink);
          store = pos < a.T;
        }
        if (store && a.dr != nullptr && kpos >= a.sink) atomicAdd(a.dr + crow + pos, dr_acc * ex2(-bk2));
      }
      int* pos_sh = reinterpret_cast<int*>(sm + k2Pos);
      if (half == 0) pos_sh[key_row] = store ? pos : -1;
      // dK (x scale) then dV, 32 columns per round: each thread stages 16 columns
      // of its key row (16-byte chunks XOR-swizzled by row), then the 256 threads
      // write rows out, eight threads per 128-byte row
      const int t2 = tid - 128, c16 = t2 & 7;
      for (int r = 0; r < 8; ++r) {
        const int c = r & 3;
        const bool is_v = r >= 4;
        uint32_t v16[16];
        tmem_ld16(lane_addr + (is_v ? k2ColDV : k2ColDK) + (uint32_t)(32 * c + 16 * half), v16);
        tmem_wait_ld();
        const float sc = is_v ? 1.f : a.scale;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int ch = (4 * half + j) ^ (key_row & 7);
          *reinterpret_cast<float4*>(sm + k2Stage + key_row * 128 + ch * 16) =
              make_float4(__uint_as_float(v16[4 * j]) * sc, __uint_as_float(v16[4 * j + 1]) * sc,
                          __uint_as_float(v16[4 * j + 2]) * sc, __uint_as_float(v16[4 * j + 3]) * sc);
        }
        bar_sync(1, 256);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int row = q * 32 + (t2 >> 3), p = pos_sh[row];
          const float4 val =
              *reinterpret_cast<const float4*>(sm + k2Stage + row * 128 + ((c16 ^ (row & 7)) * 16));
          if (p >= 0) {
            float* dst = (is_v ? a.dv : a.dk) + (((long long)b * a.T + p) * a.Hkv + h) * HD + 32 * c + 4 * c16;
            if constexpr (kColumn) atomicAdd(reinterpret_cast<float4*>(dst), val);
            else *reinterpret_cast<float4*>(dst) = val;
          }
        }
        bar_sync(1, 256);                                  // the stage may be overwritten
      }
      tc_fence_before();                                   // dK, dV read before the next item's products
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

size_t attn_backward_col_items_cap(const lte_dims* d) {
  const int G = d->Hq / d->Hkv, TOK = G > 0 && G <= bwdtc::kRowsK2 ? bwdtc::kRowsK2 / G : 1;
  const long long n_ctiles = ((long long)d->sink + d->T + bwdtc::kKeysKV - 1) / bwdtc::kKeysKV;
  const long long runs = (((long long)d->T + TOK - 1) / TOK + bwdtc::kSplitRowsK2 - 1) / bwdtc::kSplitRowsK2;
  return (size_t)d->B * d->Hkv * n_ctiles * runs;
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
    if (!encode(&mk, a.k, 4, dims, st, box) || !encode(&mv, a.v, 4, dims, st, box)) return cudaErrorInvalidValue;
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
  int dev = 0, n_sm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  // window part: item = (b, h, key tile)
  const long long n_win = (long long)((a.T + kKeysKV - 1) / kKeysKV) * a.Hkv * B;
  if (n_win > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  if (n_win > 0) {
    const int grid = (int)(n_win < n_sm ? n_win : n_sm);
    bwd_dkdv_tc_kernel<false><<<grid, kThreadsK2, k2Smem, stream>>>(mq, mdo, mk, mv, a, nullptr, nullptr,
                                                                   (int)n_win, err);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // column part: the work list, then one CTA per SM over it
  const int n_ctiles = (a.sink + a.T + kKeysKV - 1) / kKeysKV;
  const long long units = (long long)B * a.Hkv;
  if (units == 0 || n_ctiles == 0) return cudaSuccess;
  if (units > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  int* n_items = reinterpret_cast<int*>(a.col_work);
  K2Item* items = reinterpret_cast<K2Item*>(static_cast<char*>(a.col_work) + 256);
  if ((e = cudaMemsetAsync(n_items, 0, sizeof(int), stream)) != cudaSuccess) return e;
  bwd_col_items_kernel<<<(unsigned)units, kColItemsThreads, 0, stream>>>(a, n_ctiles, items, n_items);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_dkdv_tc_kernel<true><<<n_sm, kThreadsK2, k2Smem, stream>>>(mq, mdo, mkc, mvc, a, items, n_items, 0, err);
  return cudaGetLastError();
}

cudaError_t attn_backward_dq_tc(const bwd::Args& a, int B, DevError* err, cudaStream_t stream) {
  using namespace bwdtc;
  const int TOK = kRowsTc / a.G;
  // tensor maps of Q, dO, o, K, V and of the column segment (contiguous rows of
  // 128 bf16; 128-byte swizzle, 64-column boxes)
  CUtensorMap mq, mdo, mo, mk, mv, mkc, mvc;
  {
    const cuuint64_t dims[4] = {(cuuint64_t)HD, (cuuint64_t)a.Hq, (cuuint64_t)a.T, (cuuint64_t)B};
    const cuuint64_t st[3] = {(cuuint64_t)HD * 2, (cuuint64_t)a.Hq * HD * 2, (cuuint64_t)a.T * a.Hq * HD * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)a.G, (cuuint32_t)TOK, 1};
    if (!encode(&mq, a.q, 4, dims, st, box) || !encode(&mdo, a.dO, 4, dims, st, box) ||
        !encode(&mo, a.o, 4, dims, st, box))
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
  bwd_dq_tc_kernel<<<dim3(n_tiles, a.Hkv, B), kThreadsP, kSmemP, stream>>>(mq, mdo, mo, mk, mv, mkc, mvc, a, err);
  return cudaGetLastError();
}

}  // namespace lte
