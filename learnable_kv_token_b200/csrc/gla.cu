// Gated linear attention, the linear-attention layer of the laLTE hybrid.
//
// "Sparse Linear Attention: Viewing SWA from the Perspective of Linear
// Attention", section "Background: Linear attention": the state is decayed,
// the value-key outer product is written, the query reads it:
//   S_t = S_{t-1} diag(a_t) + v_t k_t^T,   o_t = S_t q_t    (S: d_v x d_k).
// The hybrid that interleaves this layer with LTE is the one of "Alleviating
// Forgetfulness of Linear Attention by Hybrid Sparse Attention and
// Contextualized Learnable Token Eviction" (TL;DR, Abstract).
//
// Prefill, chunk-wise (L = 64 tokens).  With b_t = sum_{i<=t} log a_i over
// the chunk (per key channel), m = 31 the chunk middle, S_0 the state before
// the chunk, Q~_t = q_t * e^{b_t-b_m} and K~_s = k_s * e^{b_m-b_s}:
//   o_t  = (S_0 diag(e^{b_m})) Q~_t + sum_{s<=t} (Q~_t . K~_s) v_s
//   S_L  = (S_0 diag(e^{b_m}) + sum_s v_s K~_s^T) diag(e^{b_{L-1}-b_m})
// (expanding the products gives the recurrence's S_0 diag(e^{b_{L-1}}) +
// sum_s v_s (k_s * e^{b_{L-1}-b_s})^T and S_0 (q_t * e^{b_t}); the middle
// reference halves the range of the intra-chunk factors).  The factors are
// running products of the gates (of a within the second half, of 1/a
// backwards through the first), so no logarithm or exponential is evaluated.
// One CTA per (batch, head) walks the chunks in order; the fp32 state stays
// in MMA accumulator registers for the whole sequence and a bf16 copy of
// S_0 diag(e^{b_m}) in shared memory feeds the Q~ products.  The next chunk's
// q, k, v (cp.async into the other of two shared input sets) and gates (into
// registers) load while the current chunk computes.  Per chunk: Q~ and K~
// (in place), A = Q~ K~^T masked causal (64x64), O = A V + Q~ (S_0
// diag(e^{b_m}))^T (64x128), the state update (128x128), all on m16n8k16
// bf16 MMAs with fp32 accumulation.
//
// Decode: one CTA per (batch, head) streams the 128x128 fp32 state once
// (read, decay, add the outer product, write) with 16-byte accesses and
// reduces the row-query dot products with warp shuffles.
#include <math.h>

#include "lte_common.cuh"
#include "lte_internal.h"

namespace lte {
namespace gla {

constexpr int L = 64, DK = 128, DV = 128;
constexpr int kThreads = 256;

// shared-memory layout (bytes); [rows][128] bf16 tiles have 256-byte rows with
// the 16-byte chunks XOR-swizzled by (row mod 8).  Two input sets alternate
// between chunks: while chunk c computes from set c mod 2, the copies of chunk
// c+1 land in the other set.  In a set, q becomes Q~, k becomes K~ and the
// gates a become the decay factors x_t, all in place.
constexpr uint32_t kSet = 3 * 16384 + L * DK * 4;   // one input set: q, k, v [64][128] bf16, a [64][128] fp32
constexpr uint32_t kSetQ = 0, kSetK = 16384, kSetV = 32768, kSetA = 49152;
constexpr uint32_t kA = 2 * kSet;             // masked A (bf16)      [64][64], 128-byte rows
constexpr uint32_t kSb = kA + 8192;           // S_0 diag(e^{b_m}) (bf16) [128][128]
constexpr uint32_t kLamM = kSb + 32768;       // e^{b_m} per key channel (fp32)
constexpr uint32_t kLamR = kLamM + 512;       // e^{b_last - b_m} per key channel (fp32)
constexpr uint32_t kSmem = kLamR + 512;

__device__ __forceinline__ uint32_t saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// byte offset of element (r, c) in a swizzled bf16 tile with `rowb`-byte rows
__device__ __forceinline__ uint32_t sw(int r, int c, int rowb) {
  return (uint32_t)(r * rowb + ((((c >> 3) ^ (r & 7)) & (rowb / 16 - 1)) << 4) + (c & 7) * 2);
}
__device__ __forceinline__ void ldsm4(uint32_t a, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void ldsm4t(uint32_t a, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void mma(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// 1/x by the special-function unit (rcp.approx: within 1 ulp, far below the
// bf16 rounding the decay factors feed into)
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}

// A fragment (16 x 16) from a [m][k]-stored tile (row-major A)
__device__ __forceinline__ void frag_a(uint32_t base, int rowb, int m0, int k0, int lane,
                                       uint32_t* r) {
  const int row = m0 + (lane & 7) + ((lane >> 3) & 1) * 8, col = k0 + (lane >> 4) * 8;
  ldsm4(base + sw(row, col, rowb), r);
}
// A fragment (16 x 16) from a [k][m]-stored tile (A^T in memory)
__device__ __forceinline__ void frag_a_t(uint32_t base, int rowb, int m0, int k0, int lane,
                                         uint32_t* r) {
  const int row = k0 + (lane & 7) + (lane >> 4) * 8, col = m0 + ((lane >> 3) & 1) * 8;
  ldsm4t(base + sw(row, col, rowb), r);
}
// B fragments of two n8 tiles (k16 x n16) from a [n][k]-stored tile
__device__ __forceinline__ void frag_b(uint32_t base, int rowb, int n0, int k0, int lane,
                                       uint32_t* r) {
  const int row = n0 + (lane & 7) + (lane >> 4) * 8, col = k0 + ((lane >> 3) & 1) * 8;
  ldsm4(base + sw(row, col, rowb), r);
}
// B fragments of two n8 tiles (k16 x n16) from a [k][n]-stored tile
__device__ __forceinline__ void frag_b_t(uint32_t base, int rowb, int n0, int k0, int lane,
                                         uint32_t* r) {
  const int row = k0 + (lane & 7) + ((lane >> 3) & 1) * 8, col = n0 + (lane >> 4) * 8;
  ldsm4t(base + sw(row, col, rowb), r);
}

__global__ void __launch_bounds__(kThreads, 1)
gla_prefill_kernel(int T, int H, const __nv_bfloat16* __restrict__ q,
                   const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                   const float* __restrict__ a, __nv_bfloat16* __restrict__ o,
                   float* __restrict__ state) {
  extern __shared__ __align__(128) uint8_t sm[];
  const int bh = blockIdx.x, b = bh / H, hd = bh % H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, cq = lane & 3;               // accumulator row / column pair
  const uint32_t s0 = saddr(sm);
  float* lam_m = reinterpret_cast<float*>(sm + kLamM);
  float* lam_r = reinterpret_cast<float*>(sm + kLamR);
  const long long row_stride = (long long)H * DK;        // elements between tokens
  const long long base_bh = (long long)b * T * row_stride + (long long)hd * DK;

  // ---- state: fp32 master in accumulators (warp: rows 32*(w%4)..+32, cols 64*(w/4)..+64)
  const int sm0 = (warp & 3) * 32, sn0 = (warp >> 2) * 64;
  float* st = state + (long long)bh * DV * DK;
  float sacc[2][8][4];
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int ni = 0; ni < 8; ++ni)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = sm0 + mi * 16 + gq + (e >> 1) * 8, j = sn0 + ni * 8 + cq * 2 + (e & 1);
        sacc[mi][ni][e] = st[i * DK + j];
      }

  // inputs of chunk t0 -> input set `set` (async copies, one commit group)
  auto load_qkv = [&](int t0, int set) {
    const uint32_t sb = s0 + set * kSet;
    for (int c = tid; c < L * 16; c += kThreads) {
      const int r = c >> 4, cc = (c & 15) * 8;
      const long long g = base_bh + (long long)(t0 + r) * row_stride + cc;
      cp16(sb + kSetQ + sw(r, cc, 256), q + g);
      cp16(sb + kSetK + sw(r, cc, 256), k + g);
      cp16(sb + kSetV + sw(r, cc, 256), v + g);
    }
    for (int c = tid; c < L * 32; c += kThreads) {       // gates: plain [64][128] fp32 rows
      const int r = c >> 5, cc = (c & 31) * 4;
      cp16(sb + kSetA + (r * DK + cc) * 4, a + base_bh + (long long)(t0 + r) * row_stride + cc);
    }
  };
  // gate math: thread (j, half) walks 32 tokens of key channel j
  const int j = tid & 127, half = tid >> 7;
  load_qkv(0, 0);
  asm volatile("cp.async.commit_group;\n" ::);

  for (int t0 = 0, set = 0; t0 < T; t0 += L, set ^= 1) {
    const uint32_t sq = kSetQ + set * kSet, sk = kSetK + set * kSet, sv = kSetV + set * kSet;
    // the next chunk's inputs start loading (the other set is free: the
    // previous chunk ended with a barrier)
    if (t0 + L < T) load_qkv(t0 + L, set ^ 1);
    asm volatile("cp.async.commit_group;\n" ::);
    asm volatile("cp.async.wait_group 1;\n" ::);   // this chunk's set has landed
    __syncthreads();
    // ---- decay factors x_t = e^{b_t - b_m}, written over the gates (the
    // thread reads a_i before it writes x_i).  First half (warps 0-3): the
    // product of 1/a_i over t < i <= m, built backwards from the middle;
    // second half (warps 4-7): the product of a_i over m < i <= t.
    float* X = reinterpret_cast<float*>(sm + kSetA + set * kSet);   // [64][128]
    {
      float* Xj = X + half * 32 * DK + j;        // column j of this thread's 32 rows
      float g[32];                               // this thread's 32 gates, then factors
#pragma unroll
      for (int i = 0; i < 32; ++i) g[i] = Xj[i * DK];
      float pa = 1.f;                            // running product of a
      if (half == 0) {
        float pr = 1.f;                          // running product of 1/a
#pragma unroll
        for (int i = 31; i >= 0; --i) {
          const float ai = g[i];
          g[i] = pr;
          pr *= rcp_approx(ai);
          pa *= ai;
        }
        lam_m[j] = pa;                           // e^{b_m}: product of a over the first half
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          pa *= g[i];
          g[i] = pa;
        }
        lam_r[j] = pa;                           // e^{b_last - b_m}
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) Xj[i * DK] = g[i];
    }
    __syncthreads();
    // ---- Q~ = q x_t and K~ = k / x_t in place, 8 channels (16 bytes) per access
    {
      constexpr int kItems = L * 16 / kThreads;  // (row, 16-byte group) pairs per thread
      uint4 qv[kItems], kv[kItems];
      float4 x0[kItems], x1[kItems];
#pragma unroll
      for (int it = 0; it < kItems; ++it) {
        const int c = tid + it * kThreads, r = c >> 4, g = (c & 15) * 8;
        const uint32_t o16 = sw(r, g, 256);
        qv[it] = *reinterpret_cast<const uint4*>(sm + sq + o16);
        kv[it] = *reinterpret_cast<const uint4*>(sm + sk + o16);
        x0[it] = *reinterpret_cast<const float4*>(X + r * DK + g);
        x1[it] = *reinterpret_cast<const float4*>(X + r * DK + g + 4);
      }
#pragma unroll
      for (int it = 0; it < kItems; ++it) {
        const int c = tid + it * kThreads, r = c >> 4, g = (c & 15) * 8;
        const uint32_t o16 = sw(r, g, 256);
        const float xs[8] = {x0[it].x, x0[it].y, x0[it].z, x0[it].w,
                             x1[it].x, x1[it].y, x1[it].z, x1[it].w};
        const uint32_t* qw = reinterpret_cast<const uint32_t*>(&qv[it]);
        const uint32_t* kw = reinterpret_cast<const uint32_t*>(&kv[it]);
        uint32_t qo[4], ko[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 q2 = *reinterpret_cast<const __nv_bfloat162*>(&qw[e]);
          const __nv_bfloat162 k2 = *reinterpret_cast<const __nv_bfloat162*>(&kw[e]);
          const float xa = xs[2 * e], xb = xs[2 * e + 1];
          qo[e] = pack(__low2float(q2) * xa, __high2float(q2) * xb);
          ko[e] = pack(__low2float(k2) * rcp_approx(xa), __high2float(k2) * rcp_approx(xb));
        }
        *reinterpret_cast<uint4*>(sm + sq + o16) = make_uint4(qo[0], qo[1], qo[2], qo[3]);
        *reinterpret_cast<uint4*>(sm + sk + o16) = make_uint4(ko[0], ko[1], ko[2], ko[3]);
      }
    }
    __syncthreads();
    // bf16 copy of S_0 diag(e^{b_m}) for the O product
#pragma unroll
    for (int ni = 0; ni < 8; ++ni) {
      const int jj = sn0 + ni * 8 + cq * 2;
      const float m0 = lam_m[jj], m1 = lam_m[jj + 1];
#pragma unroll
      for (int mi = 0; mi < 2; ++mi)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int i = sm0 + mi * 16 + gq + hf * 8;
          *reinterpret_cast<uint32_t*>(sm + kSb + sw(i, jj, 256)) =
              pack(sacc[mi][ni][hf * 2] * m0, sacc[mi][ni][hf * 2 + 1] * m1);
        }
    }

    // ---- A = Q~ K~^T (64 x 64), causal mask s <= t, bf16 -> shared
    {
      const int am0 = (warp & 3) * 16, an0 = (warp >> 2) * 32;
      float acc[4][4] = {};
#pragma unroll
      for (int kk = 0; kk < DK; kk += 16) {
        uint32_t fa[4];
        frag_a(s0 + sq, 256, am0, kk, lane, fa);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t fb[4];
          frag_b(s0 + sk, 256, an0 + np * 16, kk, lane, fb);
          mma(acc[np * 2], fa, fb[0], fb[1]);
          mma(acc[np * 2 + 1], fa, fb[2], fb[3]);
        }
      }
#pragma unroll
      for (int ni = 0; ni < 4; ++ni)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int t = am0 + gq + hf * 8, s = an0 + ni * 8 + cq * 2;
          const float x0 = s <= t ? acc[ni][hf * 2] : 0.f;
          const float x1 = s + 1 <= t ? acc[ni][hf * 2 + 1] : 0.f;
          *reinterpret_cast<uint32_t*>(sm + kA + sw(t, s, 128)) = pack(x0, x1);
        }
    }
    __syncthreads();

    // ---- O = A V + Q~ (S_0 diag(e^{b_m}))^T (64 x 128) -> bf16 output
    {
      const int om0 = (warp & 3) * 16, on0 = (warp >> 2) * 64;
      float acc[8][4] = {};
#pragma unroll
      for (int kk = 0; kk < L; kk += 16) {
        uint32_t fa[4];
        frag_a(s0 + kA, 128, om0, kk, lane, fa);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t fb[4];
          frag_b_t(s0 + sv, 256, on0 + np * 16, kk, lane, fb);
          mma(acc[np * 2], fa, fb[0], fb[1]);
          mma(acc[np * 2 + 1], fa, fb[2], fb[3]);
        }
      }
#pragma unroll
      for (int kk = 0; kk < DK; kk += 16) {
        uint32_t fa[4];
        frag_a(s0 + sq, 256, om0, kk, lane, fa);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t fb[4];
          frag_b(s0 + kSb, 256, on0 + np * 16, kk, lane, fb);
          mma(acc[np * 2], fa, fb[0], fb[1]);
          mma(acc[np * 2 + 1], fa, fb[2], fb[3]);
        }
      }
#pragma unroll
      for (int ni = 0; ni < 8; ++ni)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int t = om0 + gq + hf * 8, i = on0 + ni * 8 + cq * 2;
          *reinterpret_cast<uint32_t*>(o + base_bh + (long long)(t0 + t) * row_stride + i) =
              pack(acc[ni][hf * 2], acc[ni][hf * 2 + 1]);
        }
    }

    // ---- S <- (S diag(e^{b_m}) + V^T K~) diag(e^{b_last - b_m})  (128 x 128, K = 64 tokens)
    auto scale_cols = [&](const float* f) {
#pragma unroll
      for (int ni = 0; ni < 8; ++ni) {
        const int jj = sn0 + ni * 8 + cq * 2;
        const float l0 = f[jj], l1 = f[jj + 1];
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
          sacc[mi][ni][0] *= l0; sacc[mi][ni][1] *= l1;
          sacc[mi][ni][2] *= l0; sacc[mi][ni][3] *= l1;
        }
      }
    };
    scale_cols(lam_m);
#pragma unroll
    for (int kk = 0; kk < L; kk += 16) {
      uint32_t fa[2][4];
      frag_a_t(s0 + sv, 256, sm0, kk, lane, fa[0]);
      frag_a_t(s0 + sv, 256, sm0 + 16, kk, lane, fa[1]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t fb[4];
        frag_b_t(s0 + sk, 256, sn0 + np * 16, kk, lane, fb);
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
          mma(sacc[mi][np * 2], fa[mi], fb[0], fb[1]);
          mma(sacc[mi][np * 2 + 1], fa[mi], fb[2], fb[3]);
        }
      }
    }
    scale_cols(lam_r);
    __syncthreads();   // every warp is done with this chunk's tiles and S_0 copy
  }
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int ni = 0; ni < 8; ++ni)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = sm0 + mi * 16 + gq + (e >> 1) * 8, jj = sn0 + ni * 8 + cq * 2 + (e & 1);
        st[i * DK + jj] = sacc[mi][ni][e];
      }
}

// ---------------------------------------------------------------- decode
template <typename TIn>
__global__ void __launch_bounds__(256)
gla_decode_kernel(int H, const TIn* __restrict__ q, const TIn* __restrict__ k,
                  const TIn* __restrict__ v, const float* __restrict__ a, TIn* __restrict__ o,
                  float* __restrict__ state) {
  const int bh = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long vb = (long long)bh * DK;
  float q4[4], k4[4], a4[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    q4[e] = to_f32(q[vb + lane * 4 + e]);
    k4[e] = to_f32(k[vb + lane * 4 + e]);
    a4[e] = a[vb + lane * 4 + e];
  }
  float* st = state + (long long)bh * DV * DK;
  constexpr int kRows = DV / 8;                       // rows per warp
  // every row's loads first (16 x 512 B in flight per warp), then update and store
  float4 s4[kRows];
  float vi[kRows];
#pragma unroll
  for (int rr = 0; rr < kRows; ++rr) {
    const int i = warp * kRows + rr;
    s4[rr] = reinterpret_cast<const float4*>(st + (long long)i * DK)[lane];
    vi[rr] = to_f32(v[(long long)bh * DV + i]);
  }
  float d[kRows];
#pragma unroll
  for (int rr = 0; rr < kRows; ++rr) {
    const int i = warp * kRows + rr;
    float4 x = s4[rr];
    x.x = fmaf(x.x, a4[0], vi[rr] * k4[0]);
    x.y = fmaf(x.y, a4[1], vi[rr] * k4[1]);
    x.z = fmaf(x.z, a4[2], vi[rr] * k4[2]);
    x.w = fmaf(x.w, a4[3], vi[rr] * k4[3]);
    reinterpret_cast<float4*>(st + (long long)i * DK)[lane] = x;
    d[rr] = x.x * q4[0] + x.y * q4[1] + x.z * q4[2] + x.w * q4[3];
  }
  // the 16 row sums across the 32 lanes: at each step a lane keeps half of its
  // values and adds its partner's copy of them (lanes paired over bit 4, 3, 2,
  // 1, then 0 -- the same pairing tree as a plain butterfly per row)
#pragma unroll
  for (int half = kRows / 2, bit = 16; half >= 1; half >>= 1, bit >>= 1) {
    const bool upper = (lane & bit) != 0;
#pragma unroll
    for (int jj = 0; jj < half; ++jj) {
      const float send = upper ? d[jj] : d[jj + half];
      const float keep = upper ? d[jj + half] : d[jj];
      d[jj] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
    }
  }
  d[0] += __shfl_xor_sync(0xffffffffu, d[0], 1);
  // lane -> row: bits 4, 3, 2, 1 of the lane select the row's bits 3, 2, 1, 0
  if ((lane & 1) == 0) {
    const int row = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 +
                    ((lane >> 1) & 1);
    o[(long long)bh * DV + warp * kRows + row] = from_f32<TIn>(d[0]);
  }
}

}  // namespace gla

cudaError_t gla_prefill(int B, int T, int H, int dk, int dv, int dtype, const void* q,
                        const void* k, const void* v, const float* a, void* o, float* state,
                        cudaStream_t stream) {
  if (dtype != LTE_BF16 || dk != gla::DK || dv != gla::DV || T % gla::L != 0)
    return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(gla::gla_prefill_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, gla::kSmem);
  if (e != cudaSuccess) return e;
  gla::gla_prefill_kernel<<<B * H, gla::kThreads, gla::kSmem, stream>>>(
      T, H, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, a,
      (__nv_bfloat16*)o, state);
  return cudaGetLastError();
}

cudaError_t gla_decode(int B, int H, int dk, int dv, int dtype, const void* q, const void* k,
                       const void* v, const float* a, void* o, float* state,
                       cudaStream_t stream) {
  if (dk != gla::DK || dv != gla::DV) return cudaErrorNotSupported;
  if (dtype == LTE_BF16)
    gla::gla_decode_kernel<__nv_bfloat16><<<B * H, 256, 0, stream>>>(
        H, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, a,
        (__nv_bfloat16*)o, state);
  else
    gla::gla_decode_kernel<float><<<B * H, 256, 0, stream>>>(
        H, (const float*)q, (const float*)k, (const float*)v, a, (float*)o, state);
  return cudaGetLastError();
}

}  // namespace lte
