// Weight gradient of the scoring CNN's first layer on 5th-generation tensor
// cores (tcgen05 + TMEM), for bf16 keys and values, 32 hidden channels, head
// dim 128 (256 input channels).
//
// "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention
// and Contextualized Learnable Token Eviction", Abstract (the CNN is trained
// end to end) and Fig. 2 caption (the CNN over past and future keys and
// values).  With x = [k; v] and dz1 the gradient at the first layer's
// pre-activation (from the elementwise pass, cnnb_dz_kernel):
//   dw1[c][ch][kk] = sum_{b, i} dz1[b][i][c] x[b][i + kk - past1][ch]
// a reduction over all B * T positions of a KV head.  Per tile of 128
// positions and per tap kk it is one product
//   D_kk[ch][c] += X_kk^T[ch][i] DZ[i][c],   X_kk[i] = x[i + kk - past1]
// with M = 128 input channels (two halves), N = 32, K = 16 positions per MMA.
// Both operands live in shared memory in the "interleaved" layout (no
// swizzle: 16-byte core-matrix rows, one row per position), so the tap shift
// kk is a start-address offset of kk rows.  x is exact in bf16; dz1 comes as
// a bf16 hi + lo pair (relative error about 2^-17), both products accumulate
// into the same fp32 TMEM accumulators, which stay resident over all the tiles
// a CTA walks; at the end they are added to dw1 with fp32 atomics.
//
// Roles (256 threads): warps 0-3 load a tile's x rows and dz1 rows with 16-byte
// cp.async copies (rows outside the sequence read as zero) into one of two
// stages; warp 4 (one elected lane) issues the MMAs; warps 4-7 add the
// accumulators (one TMEM lane quadrant each) to dw1 at the end.  Every
// mbarrier wait is bounded; a CTA that gives up adds nothing.
#include <math.h>

#include "lte_common.cuh"
#include "lte_internal.h"
#include "tc_ptx.cuh"

namespace lte {
namespace cbt {

using namespace tc;

constexpr int kPos = 128;                 // positions per tile (K of one tile)
constexpr int kC = 32;                    // hidden channels (N)
constexpr int kCh = 256;                  // input channels (2D)
constexpr int kMaxK1 = 8;                 // taps: 2 halves x k1 x 32 TMEM columns <= 512
constexpr int kThreads = 256;
constexpr int kLoaders = 128;             // warps 0-3
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr unsigned long long kWait = 1000000000ull;

// shared-memory layout of one stage: x as [32 channel groups][R rows][8], then
// dz1 as [2 planes (hi, lo)][4 channel groups][128 rows][8]
__host__ __device__ constexpr uint32_t x_bytes(int k1) { return 32u * (kPos + k1 - 1) * 16u; }
constexpr uint32_t kDzBytes = 2u * 4u * kPos * 16u;
__host__ __device__ constexpr uint32_t stage_bytes(int k1) { return x_bytes(k1) + kDzBytes; }
__host__ __device__ constexpr uint32_t smem_bytes(int k1) { return kStages * stage_bytes(k1) + 128u; }

// no-swizzle shared-memory matrix descriptor: lbo = bytes between core matrices
// along K, sbo = bytes between core matrices along M (or N)
__device__ __forceinline__ uint64_t sdesc_ns(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// instruction descriptor, kind::f16: bf16 A and B, fp32 D, both operands MN-major
__host__ __device__ constexpr uint32_t idesc_mn(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void cpa16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cpa_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cpa_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::); }
__device__ __forceinline__ void loaders_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kLoaders) : "memory");
}

struct Args {
  int B, T, Hkv, k1, past1, n_ctas;      // n_ctas per KV head
  Strides4 s;
  const __nv_bfloat16 *k, *v;
  const __nv_bfloat16* dzp;              // dz1 planes [2][B*Hkv][T][32] (hi, lo)
  float* dw1;                            // [Hkv][32][256][k1], added to
  DevError* err;
};

__global__ void __launch_bounds__(kThreads, 1) cnnb_dw1_tc_kernel(const Args a) {
  extern __shared__ __align__(1024) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y, k1 = a.k1;
  const uint32_t sb = sa(sm);
  const uint32_t tail = sb + kStages * stage_bytes(k1);
  const uint32_t bar_full = tail, bar_empty = tail + 8 * kStages, bar_done = tail + 16 * kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kStages * stage_bytes(k1) + 64);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kStages * stage_bytes(k1) + 68);
  const int R = kPos + k1 - 1;
  // this CTA's tiles of KV head h: (sequence, 128-position block) pairs
  const int per_seq = (a.T + kPos - 1) / kPos, n_tiles = a.B * per_seq;
  const int t_lo = (int)((long long)n_tiles * blockIdx.x / a.n_ctas);
  const int t_hi = (int)((long long)n_tiles * (blockIdx.x + 1) / a.n_ctas);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 4) {
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

  if (warp < 4) {
    // ---------------------------------------------------------------- loaders
    bool ok = true;
    for (int t = t_lo, it = 0; t < t_hi && ok; ++t, ++it) {
      const int st = it % kStages, use = it / kStages;
      if (use >= 1) ok = mbar_wait_bounded(bar_empty + 8 * st, (use - 1) & 1, kWait, abort_flag, a.err, 501);
      ok = __all_sync(0xffffffffu, ok);
      loaders_sync();                                  // every loader thread saw the stage free
      if (*abort_flag) ok = false;
      if (!ok) break;
      const int b = t / per_seq, p0 = (t % per_seq) * kPos;
      const uint32_t xs = sb + st * stage_bytes(k1), dzs = xs + x_bytes(k1);
      // x rows p0 - past1 .. p0 - past1 + R - 1, 16-byte chunk g (8 channels) of row r
      const long long xrow0 = (long long)b * a.s.b + (long long)h * a.s.h;
      for (int e = tid; e < 32 * R; e += kLoaders) {      // 16 threads per k (or v) row
        const int g = e & 31, r = e >> 5;
        const int pos = p0 - a.past1 + r;
        const bool in = pos >= 0 && pos < a.T;
        const __nv_bfloat16* src = (g < 16 ? a.k : a.v) + (in ? xrow0 + (long long)pos * a.s.t : 0) +
                                   (g & 15) * 8;
        cpa16(xs + (uint32_t)(g * R + r) * 16u, src, in);
      }
      // dz1 rows p0 .. p0 + 127 of both planes
      const long long urow = (long long)(b * a.Hkv + h) * a.T;
      const long long plane = (long long)a.B * a.Hkv * a.T * kC;
      for (int e = tid; e < 2 * 4 * kPos; e += kLoaders) {  // 4 threads per 64-byte row
        const int pl = e / (4 * kPos), g = e & 3, r = (e >> 2) % kPos;
        const int pos = p0 + r;
        const bool in = pos < a.T;
        const __nv_bfloat16* src = a.dzp + pl * plane + (in ? (urow + pos) * kC : 0) + g * 8;
        cpa16(dzs + (uint32_t)((pl * 4 + g) * kPos + r) * 16u, src, in);
      }
      cpa_commit();
      cpa_wait_all();
      fence_proxy_async();                             // generic writes -> tensor-core reads
      loaders_sync();
      if (tid == 0) mbar_arrive(bar_full + 8 * st);
    }
    cpa_wait_all();
  } else {
    // ---------------------------------------------------------------- MMA issuer (warp 4)
    bool ok = true;
    if (warp == 4) {
      const uint32_t id = idesc_mn(128, kC);
      for (int t = t_lo, it = 0; t < t_hi && ok; ++t, ++it) {
        const int st = it % kStages, use = it / kStages;
        ok = __all_sync(0xffffffffu,
                        mbar_wait_bounded(bar_full + 8 * st, use & 1, kWait, abort_flag, a.err, 502));
        if (!ok) break;
        tc_fence_after();
        const uint32_t xs = sb + st * stage_bytes(k1), dzs = xs + x_bytes(k1);
        if (elect_one()) {
          for (int ks = 0; ks < kPos / 16; ++ks)
            for (int pl = 0; pl < 2; ++pl) {
              const uint64_t bdesc = sdesc_ns(dzs + (uint32_t)(pl * 4 * kPos + ks * 16) * 16u, 128u,
                                              (uint32_t)kPos * 16u);
              for (int hf = 0; hf < 2; ++hf)
                for (int kk = 0; kk < k1; ++kk) {
                  const uint64_t adesc =
                      sdesc_ns(xs + (uint32_t)(hf * 16 * R + ks * 16 + kk) * 16u, 128u, (uint32_t)R * 16u);
                  const uint32_t acc = (it > 0 || ks > 0 || pl > 0) ? 1u : 0u;
                  mma_f16(tmem + (uint32_t)((hf * k1 + kk) * kC), adesc, bdesc, id, acc);
                }
            }
          mma_commit(bar_empty + 8 * st);              // the stage may be refilled
        }
        __syncwarp();
      }
      if (elect_one()) mma_commit(bar_done);           // every product issued above has completed
      __syncwarp();
    }
    // ---------------------------------------------------------------- epilogue (warps 4-7)
    const bool any = t_hi > t_lo;
    bool fin = any && mbar_wait_bounded(bar_done, 0, kWait, abort_flag, a.err, 503);
    fin = __all_sync(0xffffffffu, fin) && *abort_flag == 0;
    if (any && !fin && warp == 4) {
      // drain: the products issued before the abort complete before TMEM is freed
      const unsigned long long t0 = gtime();
      while (!mbar_try(bar_done, 0) && gtime() - t0 < kWait) {
      }
    }
    if (fin) {
      tc_fence_after();
      const int quad = warp & 3;
      const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
      for (int hf = 0; hf < 2; ++hf) {
        const int ch = hf * 128 + quad * 32 + lane;
        for (int kk = 0; kk < k1; ++kk) {
          uint32_t r[32];
          tmem_ld32(lane_addr + (uint32_t)((hf * k1 + kk) * kC), r);
          tmem_wait_ld();
#pragma unroll 4
          for (int c = 0; c < kC; ++c)
            atomicAdd(a.dw1 + (((long long)h * kC + c) * kCh + ch) * k1 + kk, __uint_as_float(r[c]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 4)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
}

// ---------------------------------------------------------------------------
// dx = the gradient at the CNN's input, added to dk (channels < 128) and dv:
//   dx[m][ch] = sum_{kk, c} dz1[m - kk + past1][c] w1[c][ch][kk]
// Per tile of 128 positions: D[m][ch] = sum_kk DZ_kk[m][c] W_kk[c][ch], with
// M = 128 positions, N = 256 channels, K = 32 hidden channels (two K16 steps
// per tap).  DZ_kk is the dz1 tile shifted by (k1 - 1 - kk) rows (K-major,
// interleaved layout, so the shift is a start-address offset); W_kk^T[ch][c]
// lives in shared memory for the CTA's KV head as bf16 hi and lo (converted
// once).  Three products per step (hi.hi, hi.lo, lo.hi) accumulate in fp32;
// two TMEM accumulators alternate so the epilogue of one tile (TMEM -> add into
// dk, dv) overlaps the products of the next.
// Roles (384 threads): warps 0-1 load dz1 tiles (cp.async) into two stages,
// warp 2 issues the MMAs (one elected lane), warps 4-11 are the epilogue (TMEM
// lane quadrant warp % 4, column half (warp - 4) / 4).
constexpr int kDxThreads = 384;
constexpr int kDxLoaders = 64;
constexpr uint32_t kDxW = 2u * 4u * kCh * 16u;                       // one tap: hi, lo [4 cg][256][8]
__host__ __device__ constexpr uint32_t dxz_bytes(int k1) { return 2u * 4u * (kPos + k1 - 1) * 16u; }
__host__ __device__ constexpr uint32_t dx_smem_bytes(int k1) {
  return (uint32_t)k1 * kDxW + 2u * dxz_bytes(k1) + 128u;
}
__device__ __forceinline__ void dx_loaders_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kDxLoaders) : "memory");
}
// instruction descriptor, kind::f16: bf16 A and B, fp32 D, both operands K-major
__host__ __device__ constexpr uint32_t idesc_k(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

struct DxArgs {
  int B, T, Hkv, k1, past1, n_ctas;
  const __nv_bfloat16* dzp;              // dz1 planes [2][B*Hkv][T][32] (hi, lo)
  const float* w1;                       // [Hkv][32][256][k1]
  float *dk, *dv;                        // [B][T][Hkv][128], added to
  DevError* err;
};

__global__ void __launch_bounds__(kDxThreads, 1) cnnb_dx_tc_kernel(const DxArgs a) {
  extern __shared__ __align__(1024) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y, k1 = a.k1;
  const int R = kPos + k1 - 1;
  const uint32_t sb = sa(sm);
  const uint32_t zs0 = sb + (uint32_t)k1 * kDxW;                       // dz1 stages
  const uint32_t tailo = (uint32_t)k1 * kDxW + 2u * dxz_bytes(k1);
  const uint32_t tail = sb + tailo;
  // barriers: full[2], empty[2] (dz1 stages), acc_full[2], acc_empty[2] (accumulators)
  const uint32_t b_full = tail, b_empty = tail + 16, b_af = tail + 32, b_ae = tail + 48;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + tailo + 64);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + tailo + 68);
  const int per_seq = (a.T + kPos - 1) / kPos, n_tiles = a.B * per_seq;
  const int t_lo = (int)((long long)n_tiles * blockIdx.x / a.n_ctas);
  const int t_hi = (int)((long long)n_tiles * (blockIdx.x + 1) / a.n_ctas);
  const int F1 = k1 - 1 - a.past1;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_full + 8 * i, 1);
      mbar_init(b_empty + 8 * i, 1);
      mbar_init(b_af + 8 * i, 1);
      mbar_init(b_ae + 8 * i, 256);
    }
    mbar_init(tail + 72, 1);                           // all products done (teardown)
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     sa(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // the head's weights as W_kk^T[ch][c], bf16 hi and lo, interleaved K-major:
  // tap kk at kk * kDxW, plane pl at + pl * 4 * 256 * 16, byte (c / 8) * 4096 + ch * 16 + (c % 8) * 2
  {
    const float* w = a.w1 + (long long)h * kC * kCh * k1;
    for (int e = tid; e < kC * kCh * k1; e += kDxThreads) {
      const int kk = e % k1, ch = (e / k1) % kCh, c = e / (k1 * kCh);
      const float x = w[e];
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
      const uint32_t off = (uint32_t)kk * kDxW + (uint32_t)(c >> 3) * 4096u + (uint32_t)ch * 16u +
                           (uint32_t)(c & 7) * 2u;
      *reinterpret_cast<__nv_bfloat16*>(sm + off) = hi;
      *reinterpret_cast<__nv_bfloat16*>(sm + off + 4u * kCh * 16u) = lo;
    }
  }
  fence_proxy_async();                               // generic writes -> tensor-core reads
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 2) {
    // ---------------------------------------------------------------- loaders
    bool ok = true;
    for (int t = t_lo, it = 0; t < t_hi && ok; ++t, ++it) {
      const int st = it & 1, use = it >> 1;
      if (use >= 1) ok = mbar_wait_bounded(b_empty + 8 * st, (use - 1) & 1, kWait, abort_flag, a.err, 511);
      ok = __all_sync(0xffffffffu, ok);
      dx_loaders_sync();
      if (*abort_flag) ok = false;
      if (!ok) break;
      const int b = t / per_seq, p0 = (t % per_seq) * kPos;
      const uint32_t zs = zs0 + (uint32_t)st * dxz_bytes(k1);
      const long long urow = (long long)(b * a.Hkv + h) * a.T;
      const long long plane = (long long)a.B * a.Hkv * a.T * kC;
      // dz1 rows p0 - F1 .. p0 - F1 + R - 1 of both planes as [plane][cg][row][8]
      for (int e = tid; e < 2 * 4 * R; e += kDxLoaders) {
        const int g = e & 3, r = (e >> 2) % R, pl = e / (4 * R);
        const int pos = p0 - F1 + r;
        const bool in = pos >= 0 && pos < a.T;
        const __nv_bfloat16* src = a.dzp + pl * plane + (in ? (urow + pos) * kC : 0) + g * 8;
        cpa16(zs + (uint32_t)((pl * 4 + g) * R + r) * 16u, src, in);
      }
      cpa_commit();
      cpa_wait_all();
      fence_proxy_async();
      dx_loaders_sync();
      if (tid == 0) mbar_arrive(b_full + 8 * st);
    }
    cpa_wait_all();
  } else if (warp == 2) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t id = idesc_k(128, kCh);
    bool ok = true;
    for (int t = t_lo, it = 0; t < t_hi && ok; ++t, ++it) {
      const int st = it & 1, use = it >> 1;
      ok = mbar_wait_bounded(b_full + 8 * st, use & 1, kWait, abort_flag, a.err, 512);
      if (ok && use >= 1) ok = mbar_wait_bounded(b_ae + 8 * st, (use - 1) & 1, kWait, abort_flag, a.err, 513);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t zs = zs0 + (uint32_t)st * dxz_bytes(k1);
      const uint32_t d = tmem + (uint32_t)st * 256u;
      if (elect_one()) {
        bool first = true;
        for (int kk = 0; kk < k1; ++kk)
          for (int ks = 0; ks < kC / 16; ++ks)
            for (int pr = 0; pr < 3; ++pr) {       // hi.hi, hi.lo, lo.hi
              const int pa = pr == 2 ? 1 : 0, pb = pr == 1 ? 1 : 0;
              // A: dz1 plane pa, rows shifted by k1 - 1 - kk, channels 16 ks ..
              const uint64_t adesc = sdesc_ns(
                  zs + (uint32_t)((pa * 4 + 2 * ks) * R + (k1 - 1 - kk)) * 16u, (uint32_t)R * 16u, 128u);
              // B: W_kk^T plane pb, channels (K) 16 ks ..
              const uint64_t bdesc = sdesc_ns(
                  sb + (uint32_t)kk * kDxW + (uint32_t)pb * 4u * kCh * 16u + (uint32_t)(2 * ks) * 4096u,
                  4096u, 128u);
              mma_f16(d, adesc, bdesc, id, first ? 0u : 1u);
              first = false;
            }
        mma_commit(b_empty + 8 * st);                  // the dz1 stage may be refilled
        mma_commit(b_af + 8 * st);                     // the accumulator is ready
      }
      __syncwarp();
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3, half = (warp - 4) >> 2;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    bool ok = true;
    for (int t = t_lo, it = 0; t < t_hi && ok; ++t, ++it) {
      const int st = it & 1, use = it >> 1;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(b_af + 8 * st, use & 1, kWait, abort_flag, a.err, 514));
      if (!ok) break;
      tc_fence_after();
      const int b = t / per_seq, p0 = (t % per_seq) * kPos;
      const int m = p0 + quad * 32 + lane;
      float* dst = (half == 0 ? a.dk : a.dv) + (((long long)b * a.T + (m < a.T ? m : 0)) * a.Hkv + h) * 128;
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lane_addr + (uint32_t)st * 256u + (uint32_t)(half * 128 + c0), r);
        tmem_wait_ld();
        if (m < a.T) {
          float4* d4 = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float4 x = d4[e];
            x.x += __uint_as_float(r[4 * e]);
            x.y += __uint_as_float(r[4 * e + 1]);
            x.z += __uint_as_float(r[4 * e + 2]);
            x.w += __uint_as_float(r[4 * e + 3]);
            d4[e] = x;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(b_ae + 8 * st);                      // the accumulator may be overwritten
    }
  }
  // every product issued above completes before TMEM is freed
  if (warp == 2) {
    const uint32_t b_done = tail + 72;
    if (elect_one()) mma_commit(b_done);
    __syncwarp();
    const unsigned long long t0 = gtime();
    while (!mbar_try(b_done, 0) && gtime() - t0 < kWait) {
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
}

}  // namespace cbt

bool score_backward_tc_supported(const lte_dims* d, const lte_cnn* cnn) {
  return d->dtype == LTE_BF16 && d->D == 128 && cnn->c_hid == cbt::kC && cnn->k1 <= cbt::kMaxK1;
}
// dx keeps the head's weights resident: k1 taps x 32 KiB of hi and lo
bool score_backward_dx_tc_supported(const lte_dims* d, const lte_cnn* cnn) {
  return score_backward_tc_supported(d, cnn) && cbt::dx_smem_bytes(cnn->k1) <= 227u * 1024u;
}

cudaError_t score_backward_dx_tc(const lte_dims* d, const lte_cnn* cnn, const void* dz_planes,
                                 float* dk, float* dv, DevError* err, cudaStream_t stream) {
  cbt::DxArgs a{};
  a.B = d->B; a.T = d->T; a.Hkv = d->Hkv; a.k1 = cnn->k1; a.past1 = cnn->past1;
  a.dzp = (const __nv_bfloat16*)dz_planes;
  a.w1 = cnn->w1;
  a.dk = dk; a.dv = dv;
  a.err = err;
  int dev = 0, n_sm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  const int per_seq = (d->T + cbt::kPos - 1) / cbt::kPos;
  const int tiles = d->B * per_seq;
  int per_head = n_sm / d->Hkv;
  per_head = per_head < 1 ? 1 : (per_head > tiles ? tiles : per_head);
  a.n_ctas = per_head;
  const uint32_t smem = cbt::dx_smem_bytes(cnn->k1);
  if (smem > 227u * 1024u) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(cbt::cnnb_dx_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cbt::cnnb_dx_tc_kernel<<<dim3(per_head, d->Hkv), cbt::kDxThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t score_backward_dw1_tc(const lte_dims* d, const lte_cnn* cnn, const void* k,
                                  const void* v, Strides4 s, const void* dz_planes, float* dw1,
                                  DevError* err, cudaStream_t stream) {
  cbt::Args a{};
  a.B = d->B; a.T = d->T; a.Hkv = d->Hkv; a.k1 = cnn->k1; a.past1 = cnn->past1; a.s = s;
  a.k = (const __nv_bfloat16*)k; a.v = (const __nv_bfloat16*)v;
  a.dzp = (const __nv_bfloat16*)dz_planes;
  a.dw1 = dw1;
  a.err = err;
  int dev = 0, n_sm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  const int per_seq = (d->T + cbt::kPos - 1) / cbt::kPos;
  const int tiles = d->B * per_seq;
  int per_head = n_sm / d->Hkv;
  per_head = per_head < 1 ? 1 : (per_head > tiles ? tiles : per_head);
  a.n_ctas = per_head;
  const uint32_t smem = cbt::smem_bytes(cnn->k1);
  cudaError_t e = cudaFuncSetAttribute(cbt::cnnb_dw1_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cbt::cnnb_dw1_tc_kernel<<<dim3(per_head, d->Hkv), cbt::kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace lte
