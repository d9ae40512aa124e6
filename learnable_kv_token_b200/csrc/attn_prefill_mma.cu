// Prefill sparse attention, bf16 tensor-core path with warp-level mma.sync.
//
// "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention
// and Contextualized Learnable Token Eviction", Fig. 2 caption (right):
// per-head A-plus-column sparsity; row t of KV head h attends to
//   S_t = { j < s : j <= t-w } u (t-w, t] u { idx[i] : max(0, n_t-C) <= i < n_t }
// (first-C cap: i in [0, min(n_t, C)); drop-the-lowest-score cap: i < n_t with
// death[i] > n_t, the lifetimes from lte_retained_lifetimes).
//
// Design.  A CTA owns 64 query rows that share one KV head: 64/G tokens x
// the G query heads of the group, so every K/V tile it loads serves all G
// heads, and the window band it must cover is only 64/G tokens wider than w.
// Four warps own 16 rows each.  Key tiles of 64 come from up to three
// ranges: the sink slots and the retained slots of the column segment (the
// compacted rows written by lte_evict_compact, so retained keys are dense),
// and the window band of the key tensor.  Tiles are double-buffered in
// shared memory with cp.async; S = Q K^T and O += P V run on m16n8k16 bf16
// MMAs with fp32 accumulators; online softmax in the exp2 domain; a per-
// (row, key) predicate is evaluated only on tiles that are not fully inside
// every row's set.  The 16-byte chunks of every shared-memory row are XOR-
// swizzled by (row mod 8) so ldmatrix reads are bank-conflict free.
#include <math.h>

#include "lte_common.cuh"
#include "lte_internal.h"
#include "mma_sync.cuh"

namespace lte {

constexpr int kMmaRows = 64;     // query rows per CTA (tokens x heads)
constexpr int kMmaKeys = 64;     // keys per tile
constexpr int kMmaThreads = 128;

struct KeyRanges {
  int start[3], count[3];   // 0: sink slots, 1: retained slots (column segment), 2: window band
};

template <int D>
__global__ void __launch_bounds__(kMmaThreads, 2)
attn_prefill_mma_kernel(int T, int Hq, int Hkv, int sink, int window, int cap, int cap_policy,
                        float scale_log2,
                        const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                        const __nv_bfloat16* __restrict__ v, Strides4 qs, Strides4 kvs,
                        const int32_t* __restrict__ cnt, const int32_t* __restrict__ death,
                        const __nv_bfloat16* __restrict__ k_col,
                        const __nv_bfloat16* __restrict__ v_col, __nv_bfloat16* __restrict__ o,
                        Strides4 os, float* __restrict__ lse) {
  constexpr int CH = D / 8;            // 16-byte chunks per row
  constexpr int KSTEPS = D / 16;
  constexpr int DN = D / 8;            // n8 tiles over the head dim
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* q_sm = smem;                                          // [64][D]
  uint8_t* kv_sm = smem + kMmaRows * D * 2;                      // [2 stages][K,V][64][D]

  const int G = Hq / Hkv;
  const int TOK = kMmaRows / G;                                  // tokens per CTA
  const int n_tiles = (T + TOK - 1) / TOK;
  const int t0 = (n_tiles - 1 - (int)blockIdx.x) * TOK;          // heavy (late) tiles first
  const int h = blockIdx.y, b = blockIdx.z, u = b * Hkv + h;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t_last = min(t0 + TOK - 1, T - 1);
  const long long crow = (long long)u * T;
  const long long col_base = (long long)u * (sink + T);
  const bool lowest = death != nullptr;      // held set filtered by lifetime, scanned from 0

  // ---- Q tile: row rho = g*TOK + i  <-  q[b, t0+i, h*G+g, :]
  for (int i = tid; i < kMmaRows * CH; i += kMmaThreads) {
    const int rho = i / CH, c = i % CH;
    const int g = rho / TOK, tt = t0 + rho % TOK;
    const bool ok = tt < T;
    const __nv_bfloat16* src =
        q + (ok ? (long long)b * qs.b + (long long)tt * qs.t + (long long)(h * G + g) * qs.h + c * 8
                : 0);
    cp_async16(smem_u32(q_sm + swz<D>(rho, c)), src, ok);
  }
  cp_async_commit();

  // ---- key ranges of the tile
  KeyRanges kr;
  {
    const int n_first = (t0 >= window) ? held_retained(cnt[crow + t0 - window], cap, cap_policy) : 0;
    const int n_last = (t_last >= window) ? held_retained(cnt[crow + t_last - window], cap, cap_policy) : 0;
    const int lo_min = n_first - cap > 0 && !lowest ? n_first - cap : 0;
    int nsink = t_last - window + 1;
    nsink = nsink < 0 ? 0 : (nsink > sink ? sink : nsink);
    nsink = nsink > T ? T : nsink;
    const int w_lo = t0 - window + 1 > 0 ? t0 - window + 1 : 0;
    int ret_start = sink + lo_min, ret_count = n_last - lo_min > 0 ? n_last - lo_min : 0;
    if (nsink > 0 && ret_count > 0 && ret_start + ret_count <= 2 * kMmaKeys &&
        (ret_start - nsink) < kMmaKeys / 2) {
      // merge sinks and retained into one contiguous slot range (masked)
      ret_count = ret_start + ret_count;
      ret_start = 0;
      nsink = 0;
    }
    kr.start[0] = 0; kr.count[0] = nsink;
    kr.start[1] = ret_start; kr.count[1] = ret_count;
    kr.start[2] = w_lo; kr.count[2] = t_last - w_lo + 1;
  }
  int tiles_in[3], total_tiles = 0;
#pragma unroll
  for (int rg = 0; rg < 3; ++rg) {
    tiles_in[rg] = (kr.count[rg] + kMmaKeys - 1) / kMmaKeys;
    total_tiles += tiles_in[rg];
  }

  auto tile_of = [&](int it, int& rg, int& off) {
    rg = 0;
    while (rg < 2 && it >= tiles_in[rg]) { it -= tiles_in[rg]; ++rg; }
    off = it * kMmaKeys;
  };
  auto load_tile = [&](int it, int stage) {
    int rg, off;
    tile_of(it, rg, off);
    const int nk = min(kMmaKeys, kr.count[rg] - off);
    uint8_t* ks = kv_sm + stage * 2 * kMmaKeys * D * 2;
    uint8_t* vs = ks + kMmaKeys * D * 2;
    for (int i = tid; i < kMmaKeys * CH; i += kMmaThreads) {
      const int r = i / CH, c = i % CH;
      const bool ok = r < nk;
      const int key = kr.start[rg] + off + (ok ? r : 0);
      long long a;
      const __nv_bfloat16 *kb, *vb;
      if (rg == 2) {
        a = (long long)b * kvs.b + (long long)key * kvs.t + (long long)h * kvs.h + c * 8;
        kb = k; vb = v;
      } else {
        a = (col_base + key) * D + c * 8;
        kb = k_col; vb = v_col;
      }
      cp_async16(smem_u32(ks + swz<D>(r, c)), kb + (ok ? a : 0), ok);
      cp_async16(smem_u32(vs + swz<D>(r, c)), vb + (ok ? a : 0), ok);
    }
  };

  // ---- per-row data for the two rows this lane holds in the accumulators
  int t_row[2], lo_row[2], hi_row[2];
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int rho = warp * 16 + (lane >> 2) + hr * 8;
    const int tt = t0 + rho % TOK;
    t_row[hr] = tt;
    int hi = 0;
    if (tt < T && tt >= window) hi = held_retained(cnt[crow + tt - window], cap, cap_policy);
    hi_row[hr] = hi;
    lo_row[hr] = hi - cap > 0 && !lowest ? hi - cap : 0;
  }
  // tile-wide bounds for the "every row sees every key" fast path
  const int lo_all = max(lo_row[0], lo_row[1]);
  const int hi_all = min(hi_row[0], hi_row[1]);

  float o_acc[DN][4];
#pragma unroll
  for (int i = 0; i < DN; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) o_acc[i][e] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  uint32_t qf[KSTEPS][4];

  if (total_tiles > 0) load_tile(0, 0);
  cp_async_commit();

  for (int it = 0; it < total_tiles; ++it) {
    const int stage = it & 1;
    if (it + 1 < total_tiles) load_tile(it + 1, stage ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (it == 0) {
      // Q fragments, kept in registers for the whole key loop
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        const int r = warp * 16 + (lane & 15), c = ks * 2 + (lane >> 4);
        ldsm_x4(smem_u32(q_sm + swz<D>(r, c)), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
      }
    }
    int rg, off;
    tile_of(it, rg, off);
    const int key0 = kr.start[rg] + off;
    const int nk = min(kMmaKeys, kr.count[rg] - off);
    const uint8_t* ks_sm = kv_sm + stage * 2 * kMmaKeys * D * 2;
    const uint8_t* vs_sm = ks_sm + kMmaKeys * D * 2;

    // ---- S = Q K^T  (16 x 64 per warp)
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {       // pairs of n8 tiles
        const int r = np * 16 + ((lane >> 4) << 3) + (lane & 7);
        const int c = ks * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_u32(ks_sm + swz<D>(r, c)), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qf[ks], b0, b1);
        mma_bf16(s[2 * np + 1], qf[ks], b2, b3);
      }
    }

    // ---- mask (only where some key of the tile is outside some row's set)
    bool full;
    if (rg == 2) {
      // window band: key j is in (t-w, t] for both rows
      full = (nk == kMmaKeys) && key0 > max(t_row[0], t_row[1]) - window &&
             key0 + kMmaKeys - 1 <= min(t_row[0], t_row[1]);
    } else {
      full = !lowest && (nk == kMmaKeys) && key0 >= sink && (key0 - sink) >= lo_all &&
             (key0 - sink + kMmaKeys) <= hi_all;
    }
    full = __all_sync(0xffffffffu, full);
    if (!full) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int hr = e >> 1;
          const int kk = nt * 8 + ((lane & 3) << 1) + (e & 1);
          const int key = key0 + kk;
          const int tt = t_row[hr];
          bool ok = kk < nk && tt < T;
          if (ok) {
            if (rg == 2) ok = key <= tt && key > tt - window;
            else if (key < sink) ok = key <= tt - window;
            else ok = (key - sink) >= lo_row[hr] && (key - sink) < hi_row[hr] &&
                      (!lowest || __ldg(death + crow + key - sink) > hi_row[hr]);
          }
          if (!ok) s[nt][e] = -INFINITY;
        }
      }
    }

    // ---- online softmax (exp2 domain)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      mx[0] = fmaxf(mx[0], fmaxf(s[nt][0], s[nt][1]));
      mx[1] = fmaxf(mx[1], fmaxf(s[nt][2], s[nt][3]));
    }
    float corr[2], m_use[2];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 1));
      mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 2));
      const float m_new = fmaxf(m_run[hr], mx[hr] * scale_log2);
      m_use[hr] = (m_new == -INFINITY) ? 0.f : m_new;
      corr[hr] = (m_run[hr] == -INFINITY) ? 0.f : exp2f(m_run[hr] - m_use[hr]);
      m_run[hr] = m_new;
      l_run[hr] *= corr[hr];
    }
    uint32_t pf[4][4];     // P as A fragments, one per k16 step of the PV product
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hr = e >> 1;
        p[e] = exp2f(fmaf(s[nt][e], scale_log2, -m_use[hr]));   // exp2(-inf) = 0
        l_run[hr] += p[e];
      }
      pf[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(p[0], p[1]);
      pf[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(p[2], p[3]);
    }
#pragma unroll
    for (int i = 0; i < DN; ++i) {
      o_acc[i][0] *= corr[0]; o_acc[i][1] *= corr[0];
      o_acc[i][2] *= corr[1]; o_acc[i][3] *= corr[1];
    }

    // ---- O += P V
#pragma unroll
    for (int kst = 0; kst < 4; ++kst) {
#pragma unroll
      for (int dp = 0; dp < DN / 2; ++dp) {   // pairs of n8 tiles over D
        const int r = kst * 16 + (((lane >> 3) & 1) << 3) + (lane & 7);
        const int c = dp * 2 + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(vs_sm + swz<D>(r, c)), b0, b1, b2, b3);
        mma_bf16(o_acc[2 * dp], pf[kst], b0, b1);
        mma_bf16(o_acc[2 * dp + 1], pf[kst], b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // ---- epilogue
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    l_run[hr] += __shfl_xor_sync(0xffffffffu, l_run[hr], 1);
    l_run[hr] += __shfl_xor_sync(0xffffffffu, l_run[hr], 2);
  }
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int rho = warp * 16 + (lane >> 2) + hr * 8;
    const int g = rho / TOK, tt = t0 + rho % TOK;
    if (tt >= T) continue;
    const float inv = 1.f / l_run[hr];
    __nv_bfloat16* orow = o + (long long)b * os.b + (long long)tt * os.t + (long long)(h * G + g) * os.h;
#pragma unroll
    for (int i = 0; i < DN; ++i) {
      const int dcol = i * 8 + ((lane & 3) << 1);
      *reinterpret_cast<uint32_t*>(orow + dcol) =
          pack_bf16(o_acc[i][hr * 2] * inv, o_acc[i][hr * 2 + 1] * inv);
    }
    if (lse != nullptr && (lane & 3) == 0)
      lse[((long long)b * Hq + h * G + g) * T + tt] = (m_run[hr] + log2f(l_run[hr])) * 0.69314718055994531f;
  }
}

template <int D>
static cudaError_t launch_mma(const PrefillArgs& a, cudaStream_t stream) {
  const lte_dims* d = a.d;
  const int G = d->Hq / d->Hkv, TOK = kMmaRows / G;
  const size_t smem = (size_t)kMmaRows * D * 2 + 2 * 2 * (size_t)kMmaKeys * D * 2;
  cudaError_t e = cudaFuncSetAttribute(attn_prefill_mma_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((d->T + TOK - 1) / TOK, d->Hkv, d->B);
  const float scale_log2 = d->scale * 1.4426950408889634f;
  attn_prefill_mma_kernel<D><<<grid, kMmaThreads, smem, stream>>>(
      d->T, d->Hq, d->Hkv, d->sink, d->window, d->cap, d->cap_policy, scale_log2,
      (const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.k, (const __nv_bfloat16*)a.v, a.qs,
      a.kvs, a.cnt, a.death, (const __nv_bfloat16*)a.k_col, (const __nv_bfloat16*)a.v_col,
      (__nv_bfloat16*)a.o, a.os, a.lse);
  return cudaGetLastError();
}

cudaError_t attn_prefill_mma(const PrefillArgs& a, cudaStream_t stream) {
  if (a.d->D == 128) return launch_mma<128>(a, stream);
  return launch_mma<64>(a, stream);
}

}  // namespace lte

namespace lte {
// The prefill kernels need no scratch beyond the error word.
size_t attn_prefill_scratch_bytes(const lte_dims*) { return 0; }
}  // namespace lte
