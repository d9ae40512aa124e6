// Retention-score CNN tile on tensor cores (bf16 keys/values, fp32 weights).
//
// "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention
// and Contextualized Learnable Token Eviction", Fig. 2 caption: a CNN stack
// over short-range past and future context yields the retention score r_{j,h}.
//
// Layer 1 is a dense contraction once its taps are laid out as columns:
//   Z[x, n = c*k1 + kk] = sum_ch x[x][ch] * w1[c][ch][kk]          (one GEMM)
//   u[c][p]             = SiLU(b1[c] + sum_kk Z[p + kk][c*k1 + kk])  (shifted sum)
// The x rows are bf16 inputs (exact); each fp32 weight is split into
// bf16 hi + lo and both products accumulate into the same fp32 accumulator
// (relative weight error ~2^-17).  Layer 2 (c_hid -> 1, k2 taps) and the
// sigmoid run in fp32.  Every value is produced by a fixed sequence of
// instructions independent of where its token falls in the tile, so a
// token's score does not depend on the tile or the addressing mode (the
// decode step's ring or a [B,T,H,D] tensor).
//
// CTA: 320 threads (10 warps = 5 row tiles of 16 x 2 column halves of 80);
// a tile covers kScoreNT = 64 output tokens (NX = 64 + k1 + k2 - 2 <= 80 rows
// of x); supported when c_hid * k1 <= 160.
#pragma once

#include "score_cnn.cuh"

namespace lte {

constexpr int kTcThreads = 320;
constexpr int kTcRows = 80;       // x rows per tile (5 x m16)
constexpr int kTcN = 160;         // Z columns (c_hid * k1, zero padded)
constexpr int kTcKC = 64;         // input channels per weight chunk

__host__ __device__ inline bool score_tc_supported(int c_hid, int k1, int k2) {
  return c_hid * k1 <= kTcN && kScoreNT + k1 + k2 - 2 <= kTcRows;
}

// shared memory (bytes): x [80][2D] bf16 | W hi, lo [160][64] bf16 | u [c_hid][NU] fp32 |
// layer-2 weights and layer-1 biases [c_hid * (k2 + 1)] fp32; Z [160][80] fp32 reuses the x
// and W region after the GEMM.
__host__ __device__ inline size_t score_tc_smem_bytes(int D, int c_hid, int k2) {
  const size_t xw = (size_t)kTcRows * 2 * D * 2 + 2 * (size_t)kTcN * kTcKC * 2;
  const size_t z = (size_t)kTcRows * kTcN * 4;
  return (xw > z ? xw : z) + (size_t)c_hid * (kScoreNT + k2 - 1) * 4 + (size_t)c_hid * (k2 + 1) * 4;
}

namespace stc {
__device__ __forceinline__ uint32_t sa(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// 16-byte chunk c of row r in a bf16 tile with `rowb`-byte rows, XOR-swizzled by (r mod 8)
__device__ __forceinline__ uint32_t sw(int r, int c, int rowb) {
  return (uint32_t)(r * rowb + ((c ^ (r & 7)) << 4));
}
__device__ __forceinline__ void ldsm4(uint32_t a, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
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
}  // namespace stc

// Layer-2 weights and layer-1 biases of head h into shared memory (wsm:
// c_hid * (k2 + 1) floats).  Visible to the CTA after its next barrier.
__device__ __forceinline__ void score_stage_w2(const ScoreParams& p, int h, float* wsm) {
  const int nw2 = p.c_hid * p.k2;
  for (int i = threadIdx.x; i < nw2; i += blockDim.x) wsm[i] = p.w2[(long long)h * nw2 + i];
  for (int i = threadIdx.x; i < p.c_hid; i += blockDim.x) wsm[nw2 + i] = p.b1[h * p.c_hid + i];
}

constexpr int kL2Groups = 4;       // layer 2: threads per token, one channel group each

// Layers 1 (tap sum, bias, SiLU) and 2 (+ sigmoid, threshold) of a tile, after
// the GEMM, shared by every tensor-core scoring kernel so that a token's score
// is the same instruction sequence wherever it is computed.  zs holds Z
// transposed, [160 columns][R rows] (the tap sum then reads consecutive rows:
// conflict-free); u gets [c_hid][NU], NU = NT + k2 - 1; wsm holds w2 and b1 of
// head h (score_stage_w2, staged before the caller's last barrier).  Row r of Z
// is x position jb - past2 - past1 + r.  Layer 2 runs kL2Groups threads per
// token, each summing a contiguous group of hidden channels in order; the
// partial sums are added in a fixed tree order.  Writes the scores of tokens
// [jb, min(jb + NT, j_end)).  All threads call it; it begins and ends with a
// barrier.
__device__ __forceinline__ void score_tail(const ScoreParams& p, const float* zs, int R, float* us,
                                           const float* wsm, int NT, int b, int h, int jb,
                                           int j_end, int T_avail) {
  const int tid = threadIdx.x, nthreads = blockDim.x;
  const int NU = NT + p.k2 - 1, nw2 = p.c_hid * p.k2;
  const float* w2s = wsm;
  const float* b1s = wsm + nw2;
  __syncthreads();                                           // Z (and wsm) are in shared memory
  // ---- u[c][q] = SiLU(b1[c] + sum_kk Z[q + kk][c*k1 + kk]); 0 outside the tokens
  const int u0 = jb - p.past2;
  for (int i = tid; i < p.c_hid * NU; i += nthreads) {
    const int c = i / NU, q = i % NU;
    const int ug = u0 + q;
    float z = 0.f;
    for (int kk = 0; kk < p.k1; ++kk) z += zs[(c * p.k1 + kk) * R + q + kk];
    us[c * NU + q] = (ug >= 0 && ug < T_avail) ? siluf_(b1s[c] + z) : 0.f;
  }
  __syncthreads();
  // ---- layer 2 + sigmoid + threshold (fp32)
  const int per_g = (p.c_hid + kL2Groups - 1) / kL2Groups;
  for (int i0 = 0; i0 < NT * kL2Groups; i0 += nthreads) {    // uniform trip count (shuffles)
    const int i = i0 + tid;
    const int tok = i / kL2Groups, grp = i % kL2Groups;
    const bool live = i < NT * kL2Groups;
    float part = 0.f;
    if (live) {
      const int c_end = min(p.c_hid, (grp + 1) * per_g);
      for (int c = grp * per_g; c < c_end; ++c)
        for (int kk = 0; kk < p.k2; ++kk) part = fmaf(w2s[c * p.k2 + kk], us[c * NU + tok + kk], part);
    }
    // groups are lanes 4k..4k+3 of a warp: ((g0 + g1) + (g2 + g3)), the same on every lane
    part += __shfl_xor_sync(0xffffffffu, part, 1);
    part += __shfl_xor_sync(0xffffffffu, part, 2);
    const int j = jb + tok;
    if (live && grp == 0 && j < j_end) {
      const float r = sigmoidf_(p.b2[h] + part);
      if (p.win_r != nullptr) {
        p.win_r[(long long)(b * p.Hkv + h) * p.window + (j % p.window)] = r;
      } else {
        const long long o = (long long)(b * p.Hkv + h) * p.T + j;
        p.r[o] = r;
        if (p.mask) p.mask[o] = (j >= p.sink && r >= p.tau) ? 1 : 0;
      }
    }
  }
  __syncthreads();   // shared memory is reused next
}

// Scores of tokens [jb, min(jb + 64, j_end)) of unit (b, h); tokens [0, T_avail)
// exist.  Called by all kTcThreads threads (it synchronises the CTA).
template <typename KV>
__device__ __forceinline__ void score_tile_tc(const ScoreParams& p, const KV& kv, int b, int h,
                                              int jb, int j_end, int T_avail, uint8_t* smem) {
  using stc::sw;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int twoD = 2 * p.D, xrow_b = twoD * 2;               // bytes per x row
  const int NU = kScoreNT + p.k2 - 1;
  const int x0 = jb - p.past2 - p.past1;
  const int ncol = p.c_hid * p.k1;
  uint8_t* xs = smem;                                          // [80][2D] bf16
  uint8_t* whi = smem + kTcRows * xrow_b;                      // [160][64] bf16
  uint8_t* wlo = whi + kTcN * kTcKC * 2;
  float* zs = reinterpret_cast<float*>(smem);                  // [160][80] fp32 (after GEMM)
  const size_t xw = (size_t)kTcRows * xrow_b + 2 * (size_t)kTcN * kTcKC * 2;
  const size_t zb = (size_t)kTcRows * kTcN * 4;
  float* us = reinterpret_cast<float*>(smem + (xw > zb ? xw : zb));   // [c_hid][NU]
  float* wsm = us + p.c_hid * NU;                              // w2, b1 of head h
  score_stage_w2(p, h, wsm);                                   // visible after the next barrier

  // ---- x rows [x0, x0 + 80): [k; v] of existing tokens, zero elsewhere
  const int cpr = xrow_b / 16;                                 // 16-byte chunks per row
  for (int i = tid; i < kTcRows * cpr; i += kTcThreads) {
    const int r = i / cpr, c = i % cpr, xg = x0 + r;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (xg >= 0 && xg < T_avail && r < kScoreNT + p.k1 + p.k2 - 2) {
      const int e = c * 8;
      const __nv_bfloat16* src = e < p.D ? kv.krow(b, h, xg) + e : kv.vrow(b, h, xg) + (e - p.D);
      val = *reinterpret_cast<const uint4*>(src);
    }
    *reinterpret_cast<uint4*>(xs + sw(r, c, xrow_b)) = val;
  }

  // ---- Z = X (80 x 2D) . W (2D x 160), weights split hi/lo, K in chunks of 64 channels
  const int mt = warp % 5, nh = warp / 5;                      // rows 16*mt, columns 80*nh
  float acc[10][4];
#pragma unroll
  for (int i = 0; i < 10; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
  const float* w1h = p.w1 + (long long)h * p.c_hid * twoD * p.k1;
  // padding rows n >= c_hid*k1 hold zero weights for every chunk
  for (int i = tid; i < (kTcN - ncol) * kTcKC; i += kTcThreads) {
    const int n = ncol + i / kTcKC, k = i % kTcKC;
    const uint32_t off = sw(n, k >> 3, kTcKC * 2) + (k & 7) * 2;
    *reinterpret_cast<__nv_bfloat16*>(whi + off) = __float2bfloat16_rn(0.f);
    *reinterpret_cast<__nv_bfloat16*>(wlo + off) = __float2bfloat16_rn(0.f);
  }
  const int per_c = kTcKC * p.k1;
  for (int ch0 = 0; ch0 < twoD; ch0 += kTcKC) {
    __syncthreads();                                           // previous chunk consumed
    // read w1[c][ch0 + k][kk] in memory order (kk fastest), store W[c*k1 + kk][k]
    for (int i = tid; i < p.c_hid * per_c; i += kTcThreads) {
      const int c = i / per_c, rem = i % per_c, k = rem / p.k1, kk = rem % p.k1;
      const float w = w1h[((long long)c * twoD + ch0) * p.k1 + rem];
      const __nv_bfloat16 hi = __float2bfloat16_rn(w);
      const __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
      const uint32_t off = sw(c * p.k1 + kk, k >> 3, kTcKC * 2) + (k & 7) * 2;
      *reinterpret_cast<__nv_bfloat16*>(whi + off) = hi;
      *reinterpret_cast<__nv_bfloat16*>(wlo + off) = lo;
    }
    __syncthreads();
#pragma unroll
    for (int ks = 0; ks < kTcKC; ks += 16) {
      uint32_t fa[4];
      {
        const int row = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int col = (ch0 + ks) / 8 + (lane >> 4);
        stc::ldsm4(stc::sa(xs + sw(row, col, xrow_b)), fa);
      }
#pragma unroll
      for (int np = 0; np < 5; ++np) {                         // pairs of n8 tiles
        const int row = nh * 80 + np * 16 + (lane & 7) + (lane >> 4) * 8;
        const int col = ks / 8 + ((lane >> 3) & 1);
        uint32_t bh[4], bl[4];
        stc::ldsm4(stc::sa(whi + sw(row, col, kTcKC * 2)), bh);
        stc::ldsm4(stc::sa(wlo + sw(row, col, kTcKC * 2)), bl);
        stc::mma(acc[2 * np], fa, bh[0], bh[1]);
        stc::mma(acc[2 * np + 1], fa, bh[2], bh[3]);
        stc::mma(acc[2 * np], fa, bl[0], bl[1]);
        stc::mma(acc[2 * np + 1], fa, bl[2], bl[3]);
      }
    }
  }
  __syncthreads();                                             // x and W no longer read
#pragma unroll
  for (int nt = 0; nt < 10; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int row = mt * 16 + (lane >> 2) + (e >> 1) * 8;
      const int col = nh * 80 + nt * 8 + (lane & 3) * 2 + (e & 1);
      zs[col * kTcRows + row] = acc[nt][e];
    }
  score_tail(p, zs, kTcRows, us, wsm, kScoreNT, b, h, jb, j_end, T_avail);   // barrier first
}

}  // namespace lte
