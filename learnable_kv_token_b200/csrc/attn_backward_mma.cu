// Backward of the prefill sparse attention for fixed attended sets, bf16
// inputs, fp32 accumulation, warp-level tensor cores (mma.sync m16n8k16).
//
// "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention
// and Contextualized Learnable Token Eviction": Abstract (the hybrids are
// trained end to end) and Fig. 2 caption (right) for the attended sets
//   S_t = { j < s : j <= t-w } u (t-w, t] u { idx[i] : i in R_t }.
// The pages give no gradient for the eviction decisions, so the sets are held
// fixed and only the softmax attention over them is differentiated.  With P
// the softmax weights of row t (recomputed from the forward's lse), o_t the
// forward output and dO_t its incoming gradient:
//   D_t = <dO_t, o_t>,  dP = dO V^T,  dS = P * (dP - D_t),
//   dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO.
//
// Kernels, in stream order (head dim 128 runs the tcgen05 dQ and dK/dV kernels
// of attn_backward_tc.cu in place of the two warp-MMA ones):
//   bwd_delta_kernel   D_t per (row, query head) from dO and o;
//   bwd_dq_kernel      one CTA per 64 query rows (64/G tokens x the G heads of
//                      a KV head), the forward's key ranges (sink slots and
//                      retained slots of the column segment, window band of
//                      k), S = Q K^T, P, dP = dO V^T, dS, dQ += dS K;
//   bwd_dkdv_kernel    one CTA per 64-key tile and a share of the query rows
//                      that attend to it, products transposed (keys as the
//                      MMA rows): S^T = K Q^T, P^T, dV += P^T dO,
//                      dP^T = V dO^T, dS^T, dK += dS^T Q.  Launched twice:
//                      for the keys of k (window part, rows t in [j, j+w),
//                      written to dk / dv), then for the slots of the column
//                      segment (sinks and retained tokens, rows from their
//                      sink / retained conditions, added into dk / dv at their
//                      positions with fp32 atomics, since a slot's rows may
//                      be split over several CTAs).
// A position attended from the window and later from the retained segment
// so receives both contributions.  Shared-memory rows are XOR-swizzled by
// (row mod 8) in 16-byte chunks, as in the forward warp-MMA kernel.
#include <math.h>

#include "lte_common.cuh"
#include "lte_internal.h"
#include "mma_sync.cuh"
#include "attn_backward.cuh"

namespace lte {
namespace bwd {

constexpr int kRows = 64;      // query rows per tile (tokens x heads)
constexpr int kKeys = 64;      // keys per tile
constexpr int kThreads = 128;  // four warps, 16 rows (dQ) or 16 keys (dK, dV) each
constexpr int kSplitRows = 32; // row tiles per CTA of the column pass

// ---------------------------------------------------------------- D_t
template <int D>
__global__ void __launch_bounds__(256)
bwd_delta_kernel(long long rows, const __nv_bfloat16* __restrict__ o,
                 const __nv_bfloat16* __restrict__ dO, int T, int Hq, float* __restrict__ delta) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);   // (b, t, head)
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  constexpr int E = D / 32;
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < E; e += 2) {
    const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(o + row * D + lane * E + e);
    const __nv_bfloat162 y = *reinterpret_cast<const __nv_bfloat162*>(dO + row * D + lane * E + e);
    acc = fmaf(__low2float(x), __low2float(y), acc);
    acc = fmaf(__high2float(x), __high2float(y), acc);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    const int hq = (int)(row % Hq);
    const long long bt = row / Hq;
    const int t = (int)(bt % T);
    const long long b = bt / T;
    delta[(b * Hq + hq) * T + t] = acc;
  }
}

// ---------------------------------------------------------------- dQ
template <int D>
__global__ void __launch_bounds__(kThreads, 1) bwd_dq_kernel(const Args a) {
  constexpr int CH = D / 8, KSTEPS = D / 16, DN = D / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* q_sm = smem;                                   // [64][D]
  uint8_t* do_sm = q_sm + kRows * D * 2;                  // [64][D]
  uint8_t* kv_sm = do_sm + kRows * D * 2;                 // [2 stages][K, V][64][D]
  const int n_tiles = (a.T + a.TOK - 1) / a.TOK;
  const int t0 = (n_tiles - 1 - (int)blockIdx.x) * a.TOK;
  const int h = blockIdx.y, b = blockIdx.z, u = b * a.Hkv + h;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t_last = min(t0 + a.TOK - 1, a.T - 1);
  const long long crow = (long long)u * a.T;
  const long long col_base = (long long)u * (a.sink + a.T);
  const bool lowest = a.death != nullptr;

  for (int i = tid; i < kRows * CH; i += kThreads) {
    const int rho = i / CH, c = i % CH;
    const int g = rho / a.TOK, tt = t0 + rho % a.TOK;
    const bool ok = tt < a.T;
    const long long off = ok ? (((long long)b * a.T + tt) * a.Hq + h * a.G + g) * D + c * 8 : 0;
    cp_async16(smem_u32(q_sm + swz<D>(rho, c)), a.q + off, ok);
    cp_async16(smem_u32(do_sm + swz<D>(rho, c)), a.dO + off, ok);
  }
  cp_async_commit();

  // key ranges of the tile: 0 sink slots, 1 retained slots, 2 window band
  int start[3], count[3];
  {
    int lo_f, n_first, lo_l, n_last;
    row_range(a, crow, t0, lo_f, n_first);
    row_range(a, crow, t_last, lo_l, n_last);
    const int lo_min = lowest ? 0 : lo_f;
    int nsink = t_last - a.window + 1;
    nsink = nsink < 0 ? 0 : (nsink > a.sink ? a.sink : nsink);
    nsink = nsink > a.T ? a.T : nsink;
    const int w_lo = t0 - a.window + 1 > 0 ? t0 - a.window + 1 : 0;
    start[0] = 0; count[0] = nsink;
    start[1] = a.sink + lo_min; count[1] = (a.cap > 0 && n_last > lo_min) ? n_last - lo_min : 0;
    start[2] = w_lo; count[2] = t_last - w_lo + 1;
  }
  int tiles_in[3], total = 0;
#pragma unroll
  for (int rg = 0; rg < 3; ++rg) {
    tiles_in[rg] = (count[rg] + kKeys - 1) / kKeys;
    total += tiles_in[rg];
  }
  auto tile_of = [&](int it, int& rg, int& off) {
    rg = 0;
    while (rg < 2 && it >= tiles_in[rg]) { it -= tiles_in[rg]; ++rg; }
    off = it * kKeys;
  };
  auto load_tile = [&](int it, int stage) {
    int rg, off;
    tile_of(it, rg, off);
    const int nk = min(kKeys, count[rg] - off);
    uint8_t* ks = kv_sm + stage * 2 * kKeys * D * 2;
    uint8_t* vs = ks + kKeys * D * 2;
    for (int i = tid; i < kKeys * CH; i += kThreads) {
      const int r = i / CH, c = i % CH;
      const bool ok = r < nk;
      const int key = start[rg] + off + (ok ? r : 0);
      long long e;
      const __nv_bfloat16 *kb, *vb;
      if (rg == 2) {
        e = (((long long)b * a.T + key) * a.Hkv + h) * D + c * 8;
        kb = a.k; vb = a.v;
      } else {
        e = (col_base + key) * D + c * 8;
        kb = a.k_col; vb = a.v_col;
      }
      cp_async16(smem_u32(ks + swz<D>(r, c)), kb + (ok ? e : 0), ok);
      cp_async16(smem_u32(vs + swz<D>(r, c)), vb + (ok ? e : 0), ok);
    }
  };

  // the two rows this lane holds in the accumulators
  int t_row[2], lo_row[2], hi_row[2];
  float lse2[2], dl[2];
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int rho = warp * 16 + (lane >> 2) + hr * 8;
    const int g = rho / a.TOK, tt = t0 + rho % a.TOK;
    t_row[hr] = tt;
    row_range(a, crow, tt, lo_row[hr], hi_row[hr]);
    if (lowest) lo_row[hr] = 0;
    const long long li = ((long long)b * a.Hq + h * a.G + g) * a.T + tt;
    lse2[hr] = tt < a.T ? a.lse[li] * 1.4426950408889634f : 0.f;
    dl[hr] = tt < a.T ? a.delta[li] : 0.f;
  }

  float dq_acc[DN][4];
#pragma unroll
  for (int i = 0; i < DN; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dq_acc[i][e] = 0.f;

  if (total > 0) load_tile(0, 0);
  cp_async_commit();
  for (int it = 0; it < total; ++it) {
    const int stage = it & 1;
    if (it + 1 < total) load_tile(it + 1, stage ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    int rg, off;
    tile_of(it, rg, off);
    const int key0 = start[rg] + off;
    const int nk = min(kKeys, count[rg] - off);
    const uint8_t* ks_sm = kv_sm + stage * 2 * kKeys * D * 2;
    const uint8_t* vs_sm = ks_sm + kKeys * D * 2;

    // S = Q K^T and dP = dO V^T (16 x 64 per warp)
    float s[8][4], dp[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nt][e] = dp[nt][e] = 0.f;
#pragma unroll
    for (int kst = 0; kst < KSTEPS; ++kst) {
      uint32_t qa[4], da[4];
      {
        const int r = warp * 16 + (lane & 15), c = kst * 2 + (lane >> 4);
        ldsm_x4(smem_u32(q_sm + swz<D>(r, c)), qa[0], qa[1], qa[2], qa[3]);
        ldsm_x4(smem_u32(do_sm + swz<D>(r, c)), da[0], da[1], da[2], da[3]);
      }
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int r = np * 16 + ((lane >> 4) << 3) + (lane & 7);
        const int c = kst * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_u32(ks_sm + swz<D>(r, c)), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qa, b0, b1);
        mma_bf16(s[2 * np + 1], qa, b2, b3);
        ldsm_x4(smem_u32(vs_sm + swz<D>(r, c)), b0, b1, b2, b3);
        mma_bf16(dp[2 * np], da, b0, b1);
        mma_bf16(dp[2 * np + 1], da, b2, b3);
      }
    }
    // P from the forward's lse, dS = P (dP - D); masked keys give P = 0
    uint32_t dsf[4][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      float ds[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hr = e >> 1;
        const int kk = nt * 8 + ((lane & 3) << 1) + (e & 1);
        const int key = key0 + kk;
        const int tt = t_row[hr];
        bool ok = kk < nk && tt < a.T;
        if (ok) {
          if (rg == 2) ok = key <= tt && key > tt - a.window;
          else if (key < a.sink) ok = key <= tt - a.window;
          else
            ok = (key - a.sink) >= lo_row[hr] && (key - a.sink) < hi_row[hr] &&
                 (!lowest || __ldg(a.death + crow + key - a.sink) > hi_row[hr]);
        }
        const float p = ok ? exp2f(fmaf(s[nt][e], a.scale_log2, -lse2[hr])) : 0.f;
        ds[e] = p * (dp[nt][e] - dl[hr]);
      }
      dsf[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(ds[0], ds[1]);
      dsf[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(ds[2], ds[3]);
    }
    // dQ += dS K (keys as the reduction dimension)
#pragma unroll
    for (int kst = 0; kst < 4; ++kst) {
#pragma unroll
      for (int dpn = 0; dpn < DN / 2; ++dpn) {
        const int r = kst * 16 + (((lane >> 3) & 1) << 3) + (lane & 7);
        const int c = dpn * 2 + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(ks_sm + swz<D>(r, c)), b0, b1, b2, b3);
        mma_bf16(dq_acc[2 * dpn], dsf[kst], b0, b1);
        mma_bf16(dq_acc[2 * dpn + 1], dsf[kst], b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int rho = warp * 16 + (lane >> 2) + hr * 8;
    const int g = rho / a.TOK, tt = t0 + rho % a.TOK;
    if (tt >= a.T) continue;
    float* row = a.dq + (((long long)b * a.T + tt) * a.Hq + h * a.G + g) * D;
#pragma unroll
    for (int i = 0; i < DN; ++i) {
      const int dcol = i * 8 + ((lane & 3) << 1);
      *reinterpret_cast<float2*>(row + dcol) =
          make_float2(dq_acc[i][hr * 2] * a.scale, dq_acc[i][hr * 2 + 1] * a.scale);
    }
  }
}

// ---------------------------------------------------------------- dK, dV
// kColumn = false: key tile of k / v positions [j0, j0 + 64) (window part);
// kColumn = true:  slot tile [c0, c0 + 64) of the column segment, this CTA's
//                  share (blockIdx.x % n_split) of the rows that attend to it.
template <int D, bool kColumn>
__global__ void __launch_bounds__(kThreads, 1) bwd_dkdv_kernel(const Args a, int n_split) {
  constexpr int CH = D / 8, KSTEPS = D / 16, DN = D / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* k_sm = smem;                                   // [64][D]
  uint8_t* v_sm = k_sm + kKeys * D * 2;                   // [64][D]
  uint8_t* qd_sm = v_sm + kKeys * D * 2;                  // [2 stages][Q, dO][64][D]
  float* meta = reinterpret_cast<float*>(qd_sm + 2 * 2 * kRows * D * 2);   // [2][lse2, D][64]
  int* tok = reinterpret_cast<int*>(meta + 2 * 2 * kRows);                 // [2][t, lo, hi][64]
  __shared__ int range_sh[2];
  const int h = blockIdx.y, b = blockIdx.z, u = b * a.Hkv + h;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long crow = (long long)u * a.T;
  const long long col_base = (long long)u * (a.sink + a.T);
  const bool lowest = a.death != nullptr;
  const int tile = kColumn ? (int)blockIdx.x / n_split : (int)blockIdx.x;
  const int split = kColumn ? (int)blockIdx.x % n_split : 0;
  const int k0 = tile * kKeys;                            // first key position or slot
  int nk;
  if constexpr (kColumn) {
    const int n_slots = a.sink + __ldg(a.nret + u);
    nk = min(kKeys, n_slots - k0);
  } else {
    nk = min(kKeys, a.T - k0);
  }
  if (nk <= 0) return;

  // token range of the rows that attend to the tile's keys
  if (tid == 0) {
    int lo_t, hi_t;
    attending_tokens(a, crow, kColumn, k0, nk, lo_t, hi_t);
    range_sh[0] = lo_t;
    range_sh[1] = hi_t;
  }
  // K and V of the tile (resident)
  for (int i = tid; i < kKeys * CH; i += kThreads) {
    const int r = i / CH, c = i % CH;
    const bool ok = r < nk;
    long long e = 0;
    if (ok) {
      if constexpr (kColumn) e = (col_base + k0 + r) * D + c * 8;
      else e = (((long long)b * a.T + k0 + r) * a.Hkv + h) * D + c * 8;
    }
    const __nv_bfloat16* kb = kColumn ? a.k_col : a.k;
    const __nv_bfloat16* vb = kColumn ? a.v_col : a.v;
    cp_async16(smem_u32(k_sm + swz<D>(r, c)), kb + e, ok);
    cp_async16(smem_u32(v_sm + swz<D>(r, c)), vb + e, ok);
  }
  cp_async_commit();
  __syncthreads();
  int tt_lo = range_sh[0], tt_hi = range_sh[1];
  if (tt_lo > tt_hi) {                                     // no row attends (empty share)
    cp_async_wait<0>();
    return;
  }
  int rt0 = tt_lo / a.TOK, rt1 = tt_hi / a.TOK;            // row tiles [rt0, rt1]
  if constexpr (kColumn) {
    const int first = rt0 + split * kSplitRows;
    if (first > rt1) {
      cp_async_wait<0>();
      return;
    }
    rt0 = first;
    rt1 = min(rt1, first + kSplitRows - 1);
  }
  const int n_rt = rt1 - rt0 + 1;

  auto load_rows = [&](int it, int stage) {
    const int t0 = (rt0 + it) * a.TOK;
    uint8_t* qs = qd_sm + stage * 2 * kRows * D * 2;
    uint8_t* ds = qs + kRows * D * 2;
    for (int i = tid; i < kRows * CH; i += kThreads) {
      const int rho = i / CH, c = i % CH;
      const int g = rho / a.TOK, tt = t0 + rho % a.TOK;
      const bool ok = tt < a.T;
      const long long off = ok ? (((long long)b * a.T + tt) * a.Hq + h * a.G + g) * D + c * 8 : 0;
      cp_async16(smem_u32(qs + swz<D>(rho, c)), a.q + off, ok);
      cp_async16(smem_u32(ds + swz<D>(rho, c)), a.dO + off, ok);
    }
    if (tid < kRows) {
      const int rho = tid, g = rho / a.TOK, tt = t0 + rho % a.TOK;
      float* m = meta + stage * 2 * kRows;
      int* tk = tok + stage * 3 * kRows;
      const long long li = ((long long)b * a.Hq + h * a.G + g) * a.T + tt;
      m[rho] = tt < a.T ? a.lse[li] * 1.4426950408889634f : 0.f;
      m[kRows + rho] = tt < a.T ? a.delta[li] : 0.f;
      int lo, hi;
      row_range(a, crow, tt, lo, hi);
      if (lowest) lo = 0;
      tk[rho] = tt;
      tk[kRows + rho] = lo;
      tk[2 * kRows + rho] = hi;
    }
  };

  float dk_acc[DN][4], dv_acc[DN][4];
#pragma unroll
  for (int i = 0; i < DN; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk_acc[i][e] = dv_acc[i][e] = 0.f;

  load_rows(0, 0);
  cp_async_commit();
  for (int it = 0; it < n_rt; ++it) {
    const int stage = it & 1;
    if (it + 1 < n_rt) load_rows(it + 1, stage ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint8_t* qs = qd_sm + stage * 2 * kRows * D * 2;
    const uint8_t* ds_sm = qs + kRows * D * 2;
    const float* m = meta + stage * 2 * kRows;
    const int* tk = tok + stage * 3 * kRows;

    // S^T = K Q^T (16 keys x 64 rows per warp)
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
    for (int kst = 0; kst < KSTEPS; ++kst) {
      uint32_t ka[4];
      ldsm_x4(smem_u32(k_sm + swz<D>(warp * 16 + (lane & 15), kst * 2 + (lane >> 4))), ka[0], ka[1],
              ka[2], ka[3]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int r = np * 16 + ((lane >> 4) << 3) + (lane & 7);
        const int c = kst * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_u32(qs + swz<D>(r, c)), b0, b1, b2, b3);
        mma_bf16(s[2 * np], ka, b0, b1);
        mma_bf16(s[2 * np + 1], ka, b2, b3);
      }
    }
    // P^T from the forward's lse (masked pairs 0)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kl = warp * 16 + (lane >> 2) + ((e >> 1) << 3);
        const int rho = nt * 8 + ((lane & 3) << 1) + (e & 1);
        const int tt = tk[rho];
        bool ok = kl < nk && tt < a.T;
        if (ok) {
          if constexpr (!kColumn) {
            const int j = k0 + kl;
            ok = j <= tt && j > tt - a.window;
          } else {
            const int slot = k0 + kl;
            if (slot < a.sink) ok = slot <= tt - a.window;
            else {
              const int i = slot - a.sink, hi = tk[2 * kRows + rho];
              ok = i >= tk[kRows + rho] && i < hi &&
                   (!lowest || __ldg(a.death + crow + i) > hi);
            }
          }
        }
        s[nt][e] = ok ? exp2f(fmaf(s[nt][e], a.scale_log2, -m[rho])) : 0.f;
      }
    // dV += P^T dO (rows as the reduction dimension)
    {
      uint32_t pf[4][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        pf[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(s[nt][0], s[nt][1]);
        pf[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(s[nt][2], s[nt][3]);
      }
#pragma unroll
      for (int kst = 0; kst < 4; ++kst)
#pragma unroll
        for (int dpn = 0; dpn < DN / 2; ++dpn) {
          const int r = kst * 16 + (((lane >> 3) & 1) << 3) + (lane & 7);
          const int c = dpn * 2 + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(ds_sm + swz<D>(r, c)), b0, b1, b2, b3);
          mma_bf16(dv_acc[2 * dpn], pf[kst], b0, b1);
          mma_bf16(dv_acc[2 * dpn + 1], pf[kst], b2, b3);
        }
    }
    // dP^T = V dO^T, then dS^T = P^T (dP^T - D)
    float dp[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) dp[nt][e] = 0.f;
#pragma unroll
    for (int kst = 0; kst < KSTEPS; ++kst) {
      uint32_t va[4];
      ldsm_x4(smem_u32(v_sm + swz<D>(warp * 16 + (lane & 15), kst * 2 + (lane >> 4))), va[0], va[1],
              va[2], va[3]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int r = np * 16 + ((lane >> 4) << 3) + (lane & 7);
        const int c = kst * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_u32(ds_sm + swz<D>(r, c)), b0, b1, b2, b3);
        mma_bf16(dp[2 * np], va, b0, b1);
        mma_bf16(dp[2 * np + 1], va, b2, b3);
      }
    }
    {
      uint32_t dsf[4][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        float x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int rho = nt * 8 + ((lane & 3) << 1) + (e & 1);
          x[e] = s[nt][e] * (dp[nt][e] - m[kRows + rho]);
        }
        dsf[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(x[0], x[1]);
        dsf[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(x[2], x[3]);
      }
      // dK += dS^T Q
#pragma unroll
      for (int kst = 0; kst < 4; ++kst)
#pragma unroll
        for (int dpn = 0; dpn < DN / 2; ++dpn) {
          const int r = kst * 16 + (((lane >> 3) & 1) << 3) + (lane & 7);
          const int c = dpn * 2 + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(qs + swz<D>(r, c)), b0, b1, b2, b3);
          mma_bf16(dk_acc[2 * dpn], dsf[kst], b0, b1);
          mma_bf16(dk_acc[2 * dpn + 1], dsf[kst], b2, b3);
        }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // rows of dk / dv: the tile's key positions (window part, written) or the
  // positions its slots hold (column part, added)
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int kl = warp * 16 + (lane >> 2) + hr * 8;
    if (kl >= nk) continue;
    int pos;
    if constexpr (kColumn) {
      const int slot = k0 + kl;
      pos = slot < a.sink ? slot : __ldg(a.idx + crow + slot - a.sink);
      if (pos >= a.T) continue;                            // a sink slot beyond a short sequence
    } else {
      pos = k0 + kl;
    }
    const long long rowoff = (((long long)b * a.T + pos) * a.Hkv + h) * D;
#pragma unroll
    for (int i = 0; i < DN; ++i) {
      const int dcol = i * 8 + ((lane & 3) << 1);
      const float k0v = dk_acc[i][hr * 2] * a.scale, k1v = dk_acc[i][hr * 2 + 1] * a.scale;
      const float v0v = dv_acc[i][hr * 2], v1v = dv_acc[i][hr * 2 + 1];
      if constexpr (kColumn) {
        atomicAdd(a.dk + rowoff + dcol, k0v);
        atomicAdd(a.dk + rowoff + dcol + 1, k1v);
        atomicAdd(a.dv + rowoff + dcol, v0v);
        atomicAdd(a.dv + rowoff + dcol + 1, v1v);
      } else {
        *reinterpret_cast<float2*>(a.dk + rowoff + dcol) = make_float2(k0v, k1v);
        *reinterpret_cast<float2*>(a.dv + rowoff + dcol) = make_float2(v0v, v1v);
      }
    }
  }
}

template <int D>
cudaError_t launch(const Args& a, int B, bool dq_tc, DevError* err, cudaStream_t stream) {
  cudaError_t e = cudaSuccess;
  if (dq_tc) {
    // the tcgen05 dQ kernel forms D_t itself (it holds each row's dO and o) and
    // writes it for the dK/dV passes
    if ((e = attn_backward_dq_tc(a, B, err, stream)) != cudaSuccess) return e;
  } else {
    const long long rows = (long long)B * a.T * a.Hq;
    bwd_delta_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(rows, a.o, a.dO, a.T, a.Hq,
                                                                         a.delta);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t smem_dq = 2 * (size_t)kRows * D * 2 + 2 * 2 * (size_t)kKeys * D * 2;
    e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem_dq);
    if (e != cudaSuccess) return e;
    const int n_tiles = (a.T + a.TOK - 1) / a.TOK;
    bwd_dq_kernel<D><<<dim3(n_tiles, a.Hkv, B), kThreads, smem_dq, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (dq_tc) return attn_backward_dkdv_tc(a, B, err, stream);   // dK, dV on tcgen05 as well
  const size_t smem_kv = 2 * (size_t)kKeys * D * 2 + 2 * 2 * (size_t)kRows * D * 2 +
                         2 * 2 * kRows * sizeof(float) + 2 * 3 * kRows * sizeof(int);
  e = cudaFuncSetAttribute(bwd_dkdv_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem_kv);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dkdv_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem_kv);
  if (e != cudaSuccess) return e;
  const int n_ktiles = (a.T + kKeys - 1) / kKeys;
  bwd_dkdv_kernel<D, false><<<dim3(n_ktiles, a.Hkv, B), kThreads, smem_kv, stream>>>(a, 1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int n_ctiles = (a.sink + a.T + kKeys - 1) / kKeys;
  const int n_split = ((a.T + a.TOK - 1) / a.TOK + kSplitRows - 1) / kSplitRows;
  const long long gx = (long long)n_ctiles * n_split;
  if (gx > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  bwd_dkdv_kernel<D, true><<<dim3((unsigned)gx, a.Hkv, B), kThreads, smem_kv, stream>>>(a, n_split);
  return cudaGetLastError();
}

}  // namespace bwd

// D_t, then (256-aligned) the work list of the tcgen05 column pass
static size_t delta_bytes_aligned(const lte_dims* d) {
  return ((size_t)d->B * d->Hq * d->T * sizeof(float) + 255) / 256 * 256;
}
size_t attn_backward_scratch_bytes(const lte_dims* d) {
  return delta_bytes_aligned(d) + 256 + 16 * attn_backward_col_items_cap(d);
}

cudaError_t attn_backward(const BackwardArgs& g, cudaStream_t stream) {
  const lte_dims* d = g.d;
  bwd::Args a{};
  a.T = d->T; a.Hq = d->Hq; a.Hkv = d->Hkv; a.G = d->Hq / d->Hkv; a.TOK = bwd::kRows / a.G;
  a.sink = d->sink; a.window = d->window; a.cap = d->cap; a.cap_policy = d->cap_policy;
  a.scale = d->scale; a.scale_log2 = d->scale * 1.4426950408889634f;
  a.q = (const __nv_bfloat16*)g.q; a.k = (const __nv_bfloat16*)g.k;
  a.v = (const __nv_bfloat16*)g.v; a.o = (const __nv_bfloat16*)g.o;
  a.dO = (const __nv_bfloat16*)g.dO; a.k_col = (const __nv_bfloat16*)g.k_col;
  a.v_col = (const __nv_bfloat16*)g.v_col;
  a.cnt = g.cnt; a.death = g.death; a.idx = g.idx; a.nret = g.nret; a.lse = g.lse;
  a.delta = reinterpret_cast<float*>(g.scratch);
  a.col_work = static_cast<char*>(g.scratch) + delta_bytes_aligned(d);
  a.dq = g.dq; a.dk = g.dk; a.dv = g.dv;
  a.bias = g.bias; a.dr = g.dr;
  // tcgen05 kernels where they apply (head dim 128), else the warp-MMA kernels
  const bool dq_tc = attn_backward_dq_tc_supported(d);
  if ((g.bias != nullptr || g.dr != nullptr) && !dq_tc) return cudaErrorNotSupported;
  if (g.dr != nullptr) {
    const cudaError_t e = cudaMemsetAsync(g.dr, 0, (size_t)d->B * d->Hkv * d->T * sizeof(float), stream);
    if (e != cudaSuccess) return e;
  }
  if (d->D == 128) return bwd::launch<128>(a, d->B, dq_tc, g.err, stream);
  return bwd::launch<64>(a, d->B, dq_tc, g.err, stream);
}

}  // namespace lte
