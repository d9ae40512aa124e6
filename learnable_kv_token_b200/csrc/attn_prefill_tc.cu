// Prefill sparse attention on 5th-generation tensor cores (tcgen05 + TMEM +
// TMA), bf16 in, fp32 accumulate, head dim 128.
//
// "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention
// and Contextualized Learnable Token Eviction", Fig. 2 caption (right): the
// per-head A-plus-column pattern.  Row t of KV head h attends to
//   S_t = { j < s : j <= t-w } u (t-w, t] u { idx[i] : max(0, n_t-C) <= i < n_t },
//   n_t = cnt[t-w] (0 for t < w).  Under the first-C cap the retained range is
//   [0, min(n_t, C)); under the drop-the-lowest-score cap it is { i < n_t :
//   death[i] > n_t } (lifetimes from lte_retained_lifetimes): the kernel
//   instance for that policy scans retained slots from 0 and ANDs a lifetime
//   bit set into each retained tile's predicate.
//
// Work item: one (batch, KV head) unit and two consecutive 128-row Q tiles
// (each 128/G tokens x the G query heads of the group, rows token-major).
// Both Q tiles consume every K/V tile the item loads, so a K/V byte read from
// L2 serves 256 rows.  Keys come in tiles of 64 from up to three ranges: the
// sink slots and the retained slots of the column segment (compacted rows,
// contiguous) and the window band of the key tensor; every tile is one TMA box
// per 64-column half.  The kernel is persistent (one CTA per SM walks a static
// heavy-first list of items).
//
// TMEM (512 columns): for each Q tile x, S_x (64 fp32 columns; its first 32
// columns are reused for P_x as bf16 pairs), O_x (128) and Q_x (64, bf16
// pairs).  Both products read their A operand from TMEM (Q for S = Q K^T, P
// for O += P V), so shared memory only feeds K and V to the tensor core.
// Warp roles (512 threads, four warpgroups):
//   warp 0     TMA producer: the item's Q rows into one shared buffer (freed as
//              soon as they are copied into TMEM), the K and V tiles of a key
//              tile into one stage of a 4-stage ring (one barrier per stage for
//              both; a stage frees once the tile's PV MMAs have run -- each
//              MMA-warp wait is costly, so the issuer waits once per key tile);
//   warp 1     TMEM owner and MMA issuer (one elected lane).  It walks one
//              stream of key tiles across items, per tile g: PV_A(g-1), S_A(g),
//              PV_B(g-1), S_B(g), also across an item boundary, so the next
//              item's first products follow the last ones without a gap.  The
//              tensor pipe runs in issue order, so when S_x(g) has completed,
//              PV_x(g-1) has too: P_x may then be overwritten and O_x rescaled
//              without a wait;
//   warps 2-3  output stores of tiles A and B (TMA stores of the staged rows);
//   warps 4-7  softmax of tile A, warps 8-11 of tile B: one thread per row
//              reads its S row from TMEM, applies the attended-set predicate
//              (a 64-bit set of at most two column intervals), exp2 via
//              ex2.approx with the scale folded into a packed FMA, writes P
//              into TMEM, and rescales its O row only when the running max
//              grew by more than 2^8 (exact: O and l share the reference max).
//              At an item's end it hands l and the max to the epilogue through
//              shared memory and goes straight on to the next item;
//   warps 12-15 item boundaries, off the softmax path: once S_x of an item's
//              last tile has run, copy the next item's Q rows of tile x from
//              the shared buffer into TMEM; once PV_x of the last tile has run,
//              O / l -> bf16 rows staged in the (now copied) Q buffer for the
//              store warps, and lse.  The next item's first PV_x waits only for
//              O_x to have been read.
// Every mbarrier wait is bounded (1 s of global time): on expiry the CTA
// records LTE_ERR_TIMEOUT in the workspace error word, stops issuing work,
// waits (bounded) for its copies and MMAs in flight, frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "lte_common.cuh"
#include "lte_internal.h"
#include "tc_ptx.cuh"

namespace lte {
namespace tc {

constexpr int BM = 128;             // rows per Q tile (TMEM lanes)
constexpr int BN = 64;              // keys per K/V tile
constexpr int HD = 128;             // head dim
constexpr int kThreads = 512;
// register split (setmaxnreg): the launch gives 128 per thread (4 warps per
// sub-partition); warpgroup 0 (TMA, MMA, two store warps) drops to 72, the
// epilogue warpgroup to 88, and the two softmax warpgroups rise to 176:
// 4 * 72 + 4 * 88 + 8 * 176 <= 16 * 128
constexpr int kRegsLaunch = 128, kRegsIssue = 72, kRegsEpi = 88, kRegsSoftmax = 176;
static_assert(4 * kRegsIssue + 4 * kRegsEpi + 8 * kRegsSoftmax <= 16 * kRegsLaunch,
              "register split fits the launch");
constexpr uint32_t kQTile = BM * HD * 2;          // 32 KiB
constexpr uint32_t kQHalf = BM * 128;             // 64-column half of a Q tile: 16 KiB
constexpr uint32_t kQBuf = 2 * kQTile;            // tiles A and B of one item: 64 KiB
constexpr uint32_t kKV = BN * HD * 2;             // 16 KiB (K or V of one tile)
constexpr uint32_t kKVHalf = BN * 128;            // 8 KiB
constexpr int kStages = 4;                        // K/V ring depth
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKV = kQBuf;                // stage s: K at +s*32K, V at +16K
constexpr uint32_t kOffBar = kOffKV + kStages * 2 * kKV;   // 192 KiB
constexpr uint32_t kOffLM = kOffBar + 512;        // l and max per row: [item parity][tile][row][2]
constexpr uint32_t kSmemBytes = kOffLM + 2 * 2 * 128 * 8;
constexpr uint32_t kTmemCols = 512;
__host__ __device__ constexpr uint32_t col_s(int x) { return x == 0 ? 0u : 64u; }     // S (and P)
__host__ __device__ constexpr uint32_t col_o(int x) { return x == 0 ? 128u : 256u; }  // O
__host__ __device__ constexpr uint32_t col_q(int x) { return x == 0 ? 384u : 448u; }  // Q

// mbarriers: KF / KE = a K/V ring stage is full / free again (one per stage);
// LM = a tile's l and max are in shared memory (one per tile and item parity,
// so that a one-tile item cannot complete a phase before the last one was seen)
enum {
  B_QF = 0, B_QFREE = 1, B_QC = 2, B_KF = 4, B_KE = B_KF + kStages, B_SF = B_KE + kStages,
  B_PF = B_SF + 2, B_PVD = B_PF + 2, B_OE = B_PVD + 2, B_FIN = B_OE + 2, B_OST = B_FIN + 1,
  B_STG = B_OST + 2, B_LM = B_STG + 2, B_SL = B_LM + 4, kNumBars = B_SL + 2
};
// SL_x: S_x of an item's last tile has completed (one phase per item).  The
// epilogue warpgroup waits on it before it overwrites Q_x; it cannot wait on
// SF_x for that tile, since it may arrive more than one phase early, where a
// parity wait would pass on an older phase.
static_assert(8 * kNumBars + 8 <= 512, "barriers, abort flag and TMEM slot fit the tail");

struct Params {
  int T, Hq, Hkv, G, TOK, sink, window, cap, cap_policy;
  int n_pairs, n_units, n_items;
  float scale_log2;
  const int32_t* cnt;
  const int32_t* death;   // lifetimes of retained slots (drop-the-lowest-score cap), else NULL
  const float* bias;      // relaxed retention: logit offset per column-segment slot, else NULL
  int col_stride;         // slots per unit of the column segment (sink + T)
  float* lse;
  DevError* err;
};

// Columns [a, b) of a 64-key tile as a bit set (empty when b <= a).
__device__ __forceinline__ uint64_t span_bits(int a, int b) {
  a = a > 0 ? a : 0;
  b = b < BN ? b : BN;
  if (b <= a) return 0ull;
  const uint64_t ones = (b - a == 64) ? ~0ull : ((1ull << (b - a)) - 1ull);
  return ones << a;
}

// max of three fp32 values in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// ---------------------------------------------------------------- work items
struct Item {
  int b, h, u, t0, t_last;     // tokens [t0, t_last] over both Q tiles
  // key ranges: 0 sink slots, 1 retained slots (column segment), 2 window band
  int s0, c0, n0, s1, c1, n1, s2, c2, total;
  __device__ __forceinline__ void tile(int it, int& rg, int& key0, int& nk) const {
    int st, cn;
    if (it < n0) { rg = 0; st = s0; cn = c0; }
    else if (it < n0 + n1) { rg = 1; it -= n0; st = s1; cn = c1; }
    else { rg = 2; it -= n0 + n1; st = s2; cn = c2; }
    key0 = st + it * BN;
    nk = min(BN, cn - it * BN);
  }
};

// The retained counts an item's key ranges depend on, loaded one item ahead
// (each role issues the next item's loads while it works on the current one,
// so their latency never stalls the pipeline).
struct ItemCounts {
  int n_first, n_last;
};
__device__ __forceinline__ void item_tokens(const Params& p, int i, int& u, int& t0, int& t_last) {
  const int pair = p.n_pairs - 1 - i / p.n_units;   // late (heavy) tokens first
  u = i % p.n_units;
  t0 = pair * 2 * p.TOK;
  t_last = min(t0 + 2 * p.TOK - 1, p.T - 1);
}
__device__ __forceinline__ ItemCounts load_counts(const Params& p, int i) {
  ItemCounts c{0, 0};
  if (i >= p.n_items) return c;
  int u, t0, t_last;
  item_tokens(p, i, u, t0, t_last);
  const long long crow = (long long)u * p.T;
  if (t0 >= p.window) c.n_first = held_retained(__ldg(p.cnt + crow + t0 - p.window), p.cap, p.cap_policy);
  if (t_last >= p.window) c.n_last = held_retained(__ldg(p.cnt + crow + t_last - p.window), p.cap, p.cap_policy);
  return c;
}
__device__ __forceinline__ Item make_item(const Params& p, int i, const ItemCounts& c) {
  Item m;
  item_tokens(p, i, m.u, m.t0, m.t_last);
  m.b = m.u / p.Hkv;
  m.h = m.u % p.Hkv;
  const int n_first = c.n_first, n_last = c.n_last;
  const int lo_min = n_first - p.cap > 0 && p.death == nullptr ? n_first - p.cap : 0;
  int nsink = m.t_last - p.window + 1;
  nsink = nsink < 0 ? 0 : (nsink > p.sink ? p.sink : nsink);
  nsink = nsink > p.T ? p.T : nsink;
  int r_start = p.sink + lo_min, r_count = (p.cap > 0 && n_last > lo_min) ? n_last - lo_min : 0;
  if (nsink > 0 && r_count > 0 && r_start - nsink < BN / 2) {   // one slot range [0, end)
    r_count += r_start;
    r_start = 0;
    nsink = 0;
  }
  const int w_lo = m.t0 - p.window + 1 > 0 ? m.t0 - p.window + 1 : 0;
  m.s0 = 0; m.c0 = nsink; m.n0 = (nsink + BN - 1) / BN;
  m.s1 = r_start; m.c1 = r_count; m.n1 = (r_count + BN - 1) / BN;
  m.s2 = w_lo; m.c2 = m.t_last - w_lo + 1;
  m.total = m.n0 + m.n1 + (m.c2 + BN - 1) / BN;
  return m;
}

// Retained slots i = i0 + c (c < 64) held at count n: 0 <= i < n and death[i] > n.
__device__ __forceinline__ uint64_t alive_bits(const int32_t* __restrict__ death_u, int i0, int n) {
  uint64_t bits = 0ull;
#pragma unroll 8
  for (int c = 0; c < BN; ++c) {
    const int i = i0 + c;
    if (i >= 0 && i < n && __ldg(death_u + i) > n) bits |= 1ull << c;
  }
  return bits;
}

// kRelax: relaxed retention for training -- every retained-segment key's
// logit gains log r (p.bias, in units of the raw score q.k), so its softmax
// weight is scaled by r; window and sink keys are unchanged.
template <bool kLowest, bool kRelax>
__global__ void __launch_bounds__(kThreads, 1)
attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_kc,
                       const __grid_constant__ CUtensorMap tm_vc,
                       const __grid_constant__ CUtensorMap tm_o, const Params p) {
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
  if (tid == 0) {
    mbar_init(bar(B_QF), 1);
    mbar_init(bar(B_QFREE), 256);
    for (int st = 0; st < kStages; ++st) {
      mbar_init(bar(B_KF + st), 1);
      mbar_init(bar(B_KE + st), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(B_QC + x), 128);
      mbar_init(bar(B_SF + x), 1);
      mbar_init(bar(B_PF + x), 128);
      mbar_init(bar(B_PVD + x), 1);
      mbar_init(bar(B_OE + x), 128);
    }
    mbar_init(bar(B_FIN), 1);
    mbar_init(bar(B_OST), 1);
    mbar_init(bar(B_OST + 1), 1);
    mbar_init(bar(B_STG), 128);
    mbar_init(bar(B_STG + 1), 128);
    for (int i = 0; i < 4; ++i) mbar_init(bar(B_LM + i), 128);
    mbar_init(bar(B_SL), 1);
    mbar_init(bar(B_SL + 1), 1);
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

  if (warp < 4) {
    // warpgroup 0: its registers go to the softmax warpgroups
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsIssue));
    if (warp == 0) {
      // ============================================================ TMA producer
      // (all 32 lanes run the loop and wait; one elected lane issues)
      int g = 0, it = 0, issued_k = 0, issued_q = 0;
      bool ok = true;
      ItemCounts cn = load_counts(p, blockIdx.x);
      for (int i = blockIdx.x; ok && i < p.n_items; i += gridDim.x, ++it) {
        const Item m = make_item(p, i, cn);
        cn = load_counts(p, i + gridDim.x);
        // the shared Q buffer is free once both softmax groups copied the last item's rows
        // out of it and the output store staged in it two items back has been read
        if (it >= 1 && !(ok = wwait(bar(B_QFREE), (it - 1) & 1, abort_flag, p.err, 201))) break;
        if (it >= 2 && !((ok = wwait(bar(B_OST), (it - 2) & 1, abort_flag, p.err, 204)) &&
                         (ok = wwait(bar(B_OST + 1), (it - 2) & 1, abort_flag, p.err, 204))))
          break;
        if (elect_one()) {
          mbar_expect_tx(bar(B_QF), kQBuf);
          for (int x = 0; x < 2; ++x)
            for (int hf = 0; hf < 2; ++hf)
              tma_load_4d(sbase + kOffQ + x * kQTile + hf * kQHalf, &tm_q, bar(B_QF), hf * 64,
                          m.h * p.G, m.t0 + x * p.TOK, m.b);
        }
        __syncwarp();
        issued_q = it + 1;
        for (int j = 0; j < m.total; ++j, ++g) {
          const int st = g % kStages, use = g / kStages;
          int rg, key0, nk;
          m.tile(j, rg, key0, nk);
          const uint32_t kd = sbase + kOffKV + st * 2 * kKV, vd = kd + kKV;
          if (use >= 1 && !(ok = wwait(bar(B_KE + st), (use - 1) & 1, abort_flag, p.err, 202)))
            break;
          if (elect_one()) {
            mbar_expect_tx(bar(B_KF + st), 2 * kKV);
            for (int hf = 0; hf < 2; ++hf) {
              if (rg == 2) {
                tma_load_4d(kd + hf * kKVHalf, &tm_k, bar(B_KF + st), hf * 64, m.h, key0, m.b);
                tma_load_4d(vd + hf * kKVHalf, &tm_v, bar(B_KF + st), hf * 64, m.h, key0, m.b);
              } else {
                tma_load_3d(kd + hf * kKVHalf, &tm_kc, bar(B_KF + st), hf * 64, key0, m.u);
                tma_load_3d(vd + hf * kKVHalf, &tm_vc, bar(B_KF + st), hf * 64, key0, m.u);
              }
            }
          }
          __syncwarp();
          issued_k = g + 1;
        }
      }
      // drain: every issued copy has landed before the CTA may exit
      if (issued_q > 0) mbar_drain(bar(B_QF), (issued_q - 1) & 1);
      for (int q = issued_k - kStages > 0 ? issued_k - kStages : 0; q < issued_k; ++q)
        mbar_drain(bar(B_KF + q % kStages), (q / kStages) & 1);

    } else if (warp == 1) {
      // ============================================================ MMA issuer
      // (all 32 lanes run the loop and wait; one elected lane issues)
      constexpr uint32_t idS = idesc(BM, BN, false);
      constexpr uint32_t idO = idesc(BM, HD, true);
      // descriptors are built once; the start-address field (addr >> 4, low
      // 14 bits) is then advanced by plain adds (shared addresses < 256 KiB)
      const uint64_t dk0 = sdesc(sbase + kOffKV, 16, 1024);
      const uint64_t dv0 = sdesc(sbase + kOffKV + kKV, kKVHalf, 1024);
      bool ok = true;
      // PV_x of global tile g (tile j of item `item`): O_x += P_x V
      auto issue_pv = [&](int x, int g, int j, int item) -> bool {
        if (!wwait(bar(B_PF + x), g & 1, abort_flag, p.err, 215)) return false;
        if (j == 0 && item >= 1 && !wwait(bar(B_OE + x), (item - 1) & 1, abort_flag, p.err, 216))
          return false;                               // the epilogue has read the previous O_x
        tc_fence_after();
        const uint64_t dv = dv0 + (((g % kStages) * 2 * kKV) >> 4);
        const uint32_t tp = tmem + col_s(x), dO = tmem + col_o(x);
        if (elect_one()) {
  #pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            mma_f16_ts(dO, tp + 8 * kk, dv + ((kk * 2048) >> 4), idO, (j > 0 || kk > 0) ? 1u : 0u);
        }
        __syncwarp();
        return true;
      };
      // key tile g is tile j of item `it`; tile g - 1 is tile jp of item itp
      int g = 0, it = 0, prev_total = 0;
      ItemCounts cn = load_counts(p, blockIdx.x);
      for (int i = blockIdx.x; ok && i < p.n_items; i += gridDim.x, ++it) {
        const Item m = make_item(p, i, cn);
        cn = load_counts(p, i + gridDim.x);
        for (int j = 0; j < m.total && ok; ++j, ++g) {
          const int st = g % kStages;
          if (!(ok = wwait(bar(B_KF + st), (g / kStages) & 1, abort_flag, p.err, 212))) break;
          const uint64_t dk = dk0 + ((st * 2 * kKV) >> 4);
          const int jp = j >= 1 ? j - 1 : prev_total - 1, itp = j >= 1 ? it : it - 1;
          for (int x = 0; x < 2 && ok; ++x) {
            if (g >= 1) {
              if (!(ok = issue_pv(x, g - 1, jp, itp))) break;
              if (j == 0 && elect_one()) mma_commit(bar(B_PVD + x));   // item itp's O_x is final
              __syncwarp();
            }
            if (j == 0 && !(ok = wwait(bar(B_QC + x), it & 1, abort_flag, p.err, 213))) break;
            tc_fence_after();
            const uint32_t tq = tmem + col_q(x), ds = tmem + col_s(x);
            if (elect_one()) {
  #pragma unroll
              for (int kk = 0; kk < HD / 16; ++kk) {
                const uint32_t offk = ((kk >> 2) * kKVHalf + (kk & 3) * 32) >> 4;
                mma_f16_ts(ds, tq + 8 * kk, dk + offk, idS, kk > 0);
              }
              mma_commit(bar(B_SF + x));
              if (j == m.total - 1) mma_commit(bar(B_SL + x));   // Q_x of this item is done with
            }
            __syncwarp();
          }
          if (!ok) break;
          if (g >= 1 && elect_one()) mma_commit(bar(B_KE + (g - 1) % kStages));   // tile g-1 done
          __syncwarp();
        }
        prev_total = m.total;
      }
      // the last tile: PV_A, PV_B, then the epilogue signals
      if (ok && g >= 1) {
        for (int x = 0; x < 2 && ok; ++x) {
          if (!(ok = issue_pv(x, g - 1, prev_total - 1, it - 1))) break;
          if (elect_one()) mma_commit(bar(B_PVD + x));
          __syncwarp();
        }
        if (ok && elect_one()) mma_commit(bar(B_KE + (g - 1) % kStages));
        __syncwarp();
      }
      if (elect_one()) mma_commit(bar(B_FIN));       // all MMAs of this warp are complete
      __syncwarp();
      mbar_drain(bar(B_FIN), 0);
    } else {
      // ============================================================ output stores
      // warp 2 stores tile A, warp 3 tile B: once all 128 rows of the tile are
      // staged in its region of the Q buffer, one TMA store per 64-column half
      // (rows past T are clipped by the copy); the region is released for the
      // next Q load when the store has read it.  Keeping this wait off the
      // softmax warps keeps their next tile on time.
      const int x = warp - 2;
      int it = 0;
      for (int i = blockIdx.x; i < p.n_items; i += gridDim.x, ++it) {
        int u, t0, t_last;
        item_tokens(p, i, u, t0, t_last);
        if (!wwait(bar(B_STG + x), it & 1, abort_flag, p.err, 225)) break;
        if (elect_one()) {
          const uint32_t src = sbase + kOffQ + x * kQTile;
          const int b = u / p.Hkv, h = u % p.Hkv;
          tma_store_4d(&tm_o, src, 0, h * p.G, t0 + x * p.TOK, b);
          tma_store_4d(&tm_o, src + kQHalf, 64, h * p.G, t0 + x * p.TOK, b);
          bulk_commit();
          bulk_wait_read();                          // staging rows read: the buffer may be reloaded
          mbar_arrive(bar(B_OST + x));
        }
        __syncwarp();
      }
      if (elect_one()) bulk_wait_all();            // output stores complete before exit
      __syncwarp();
    }
  } else if (warp < 12) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ============================================================ softmax
    const int x = (warp - 4) >> 2;                 // Q tile of this warpgroup
    const int quad = warp & 3;                     // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t colS = col_s(x), colO = col_o(x);
    float2* lm = reinterpret_cast<float2*>(smem + kOffLM) + x * 128 + row;   // + 256 * parity
    int g0 = 0, it = 0;
    bool ok = true;
    // this row's retained count n_t = cnt[t - w] of item i (0 if none), loaded one item ahead
    auto row_count = [&](int i) -> int {
      if (i >= p.n_items) return 0;
      int u, t0, t_last;
      item_tokens(p, i, u, t0, t_last);
      const int t = t0 + x * p.TOK + row / p.G;
      return (t < p.T && t >= p.window)
                 ? held_retained(__ldg(p.cnt + (long long)u * p.T + t - p.window), p.cap, p.cap_policy)
                 : 0;
    };
    ItemCounts cn = load_counts(p, blockIdx.x);
    int hi_next = row_count(blockIdx.x);
    for (int i = blockIdx.x; ok && i < p.n_items; i += gridDim.x, ++it) {
      const Item m = make_item(p, i, cn);
      const int hi_t = hi_next;
      cn = load_counts(p, i + gridDim.x);
      hi_next = row_count(i + gridDim.x);
      const int tt = m.t0 + x * p.TOK + row / p.G;
      const bool row_ok = tt < p.T;
      const int lo_t = hi_t - p.cap > 0 && !kLowest ? hi_t - p.cap : 0;
      // attended-set predicate of tile j as a bit set over its columns: the
      // window band is one interval; a slot tile holds the visible sinks and
      // the retained slots [lo_t, hi_t), two intervals.  It does not depend on
      // S, so each tile's set is built while the warp waits for that S.
      auto tile_bits = [&](int j) -> uint64_t {
        int rg, key0, nk;
        m.tile(j, rg, key0, nk);
        if (!row_ok) return 0ull;
        if (rg == 2) return span_bits(tt - p.window + 1 - key0, min(nk, tt - key0 + 1));
        const int sink_end = min(p.sink, tt - p.window + 1);
        uint64_t ret = span_bits(p.sink + lo_t - key0, min(nk, p.sink + hi_t - key0));
        if constexpr (kLowest) {
          if (ret != 0ull) ret &= alive_bits(p.death + (long long)m.u * p.T, key0 - p.sink, hi_t);
        }
        return span_bits(-key0, min(nk, sink_end - key0)) | ret;
      };
      float m_ref = -INFINITY, l_sum = 0.f;
      for (int j = 0; j < m.total; ++j) {
        const int g = g0 + j;
        uint32_t b0, b1;
        {
          const uint64_t bits = tile_bits(j);
          b0 = (uint32_t)bits;
          b1 = (uint32_t)(bits >> 32);
        }
        asm volatile("" : "+r"(b0), "+r"(b1));     // computed before the wait below
        ok = mbar_wait(bar(B_SF + x), g & 1, abort_flag, p.err, 221);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;     // tcgen05.ld is warp-collective
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32(lane_addr + colS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(lane_addr + colS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_wait_ld();
        float s[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(sr[c]);
        if constexpr (kRelax) {
          int rg, key0, nk;
          m.tile(j, rg, key0, nk);
          if (rg != 2) {                           // column-segment slots: + log r (0 on sinks)
            const float* brow = p.bias + (long long)m.u * p.col_stride + key0;   // padded by 64
#pragma unroll
            for (int c = 0; c < 64; ++c) s[c] += __ldg(brow + c);
          }
        }
        if ((b0 & b1) != ~0u) {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            if (!((b0 >> c) & 1u)) s[c] = -INFINITY;
            if (!((b1 >> c) & 1u)) s[32 + c] = -INFINITY;
          }
        }
        float m8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {              // columns e, e + 8, ..., e + 56
          m8[e] = fmax3(s[e], s[8 + e], s[16 + e]);
          m8[e] = fmax3(m8[e], s[24 + e], s[32 + e]);
          m8[e] = fmax3(m8[e], s[40 + e], s[48 + e]);
          m8[e] = fmaxf(m8[e], s[56 + e]);
        }
        float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        mx *= p.scale_log2;                        // scale > 0: max commutes with it
        const bool need = mx > m_ref + 8.f;        // lazy rescale (x256 headroom)
        float corr = 1.f;
        if (need) {
          corr = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - mx);
          m_ref = mx;
          l_sum *= corr;
        }
        // S_x(g) has completed, hence so has PV_x(g-1): O_x is current and P_x is free
        if (__any_sync(0xffffffffu, need && corr != 0.f)) {
#pragma unroll 1
          for (int c0 = 0; c0 < HD; c0 += 32) {
            uint32_t orr[32];
            tmem_ld32(lane_addr + colO + c0, orr);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * corr);
            tmem_st32(lane_addr + colO + c0, orr);
          }
          tmem_wait_st();
        }
        const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 nm2 = make_float2(-mu, -mu);
        float2 acc2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                          make_float2(0.f, 0.f)};
        uint32_t pk[32];
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2) {
          float2 z = __ffma2_rn(make_float2(s[2 * c2], s[2 * c2 + 1]), sc2, nm2);
          z.x = ex2(z.x);
          z.y = ex2(z.y);
          acc2[c2 & 3] = __fadd2_rn(acc2[c2 & 3], z);
          __nv_bfloat162 v2 = __floats2bfloat162_rn(z.x, z.y);
          pk[c2] = *reinterpret_cast<uint32_t*>(&v2);
        }
        tmem_st32(lane_addr + colS, pk);           // P_x over the first 32 columns of S_x
        const float2 a01 = __fadd2_rn(acc2[0], acc2[1]), a23 = __fadd2_rn(acc2[2], acc2[3]);
        const float2 a = __fadd2_rn(a01, a23);
        l_sum += a.x + a.y;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_PF + x));
      }
      if (!ok) break;
      // the item's l and max for the epilogue warpgroup (slot and barrier of this item's parity)
      lm[256 * (it & 1)] = make_float2(l_sum, m_ref);
      mbar_arrive(bar(B_LM + 2 * x + (it & 1)));
      g0 += m.total;
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
    // ============================================================ item boundaries
    const int quad = warp & 3;                     // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const int g_in_row = row % p.G;
    const float2* lm = reinterpret_cast<const float2*>(smem + kOffLM) + row;
    // copy this thread's row of Q tile x from the shared buffer (128B-swizzled
    // halves) into TMEM; the caller has seen the buffer's Q copy land
    auto copy_q = [&](int x) {
      const uint8_t* qrow = smem + kOffQ + x * kQTile + row * 128;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t r[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v4 = *reinterpret_cast<const uint4*>(qrow + hf * kQHalf + ((c ^ (row & 7)) << 4));
          r[4 * c] = v4.x; r[4 * c + 1] = v4.y; r[4 * c + 2] = v4.z; r[4 * c + 3] = v4.w;
        }
        tmem_st32(lane_addr + col_q(x) + hf * 32, r);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_QC + x));
      mbar_arrive(bar(B_QFREE));
    };
    int it = 0;
    bool ok = true;
    if (blockIdx.x < p.n_items) {
      ok = wwait(bar(B_QF), 0, abort_flag, p.err, 224);
      if (ok) {
        copy_q(0);
        copy_q(1);
      }
    }
    ItemCounts cn = load_counts(p, blockIdx.x);
    for (int i = blockIdx.x; ok && i < p.n_items; i += gridDim.x, ++it) {
      const Item m = make_item(p, i, cn);
      cn = load_counts(p, i + gridDim.x);
      // the next item's Q: tile x's rows go into TMEM once S_x of this item's last
      // tile has run (Q_x is no longer read), overlapping that tile's softmax
      if (i + (int)gridDim.x < p.n_items) {
        if (!(ok = wwait(bar(B_QF), (it + 1) & 1, abort_flag, p.err, 224))) break;
        for (int x = 0; x < 2 && ok; ++x) {
          if (!(ok = wwait(bar(B_SL + x), it & 1, abort_flag, p.err, 226))) break;
          tc_fence_after();
          copy_q(x);
        }
        if (!ok) break;
      }
      // ---- epilogue: O / l -> bf16 rows staged in tile x's region of the Q
      // buffer (the next item's rows have been copied out of it, and the store
      // of the previous item has read it), then warp 2 + x stores them; rows
      // past T are clipped by the copy
      for (int x = 0; x < 2 && ok; ++x) {
        if (!(ok = wwait(bar(B_LM + 2 * x + (it & 1)), (it >> 1) & 1, abort_flag, p.err, 227)))
          break;
        if (!(ok = wwait(bar(B_PVD + x), it & 1, abort_flag, p.err, 223))) break;
        if (it >= 1 && !(ok = wwait(bar(B_OST + x), (it - 1) & 1, abort_flag, p.err, 228))) break;
        tc_fence_after();
        const float2 lmv = lm[256 * (it & 1) + 128 * x];
        const float l_sum = lmv.x, m_ref = lmv.y;
        const float inv = __frcp_rn(l_sum);
        uint8_t* srow = smem + kOffQ + x * kQTile + row * 128;
#pragma unroll 1
        for (int c0 = 0; c0 < HD; c0 += 32) {      // 32 columns per wait
          uint32_t orr[32];
          tmem_ld32(lane_addr + col_o(x) + c0, orr);
          tmem_wait_ld();
          uint8_t* half = srow + (c0 >> 6) * kQHalf;
#pragma unroll
          for (int e = 0; e < 4; ++e) {             // 16-byte chunk (c0 % 64) / 8 + e of the half row
            uint4 v;
            uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(orr[8 * e + 2 * f]) * inv,
                                                        __uint_as_float(orr[8 * e + 2 * f + 1]) * inv);
              w[f] = *reinterpret_cast<uint32_t*>(&v2);
            }
            const int chunk = ((c0 & 63) >> 3) + e;
            *reinterpret_cast<uint4*>(half + ((chunk ^ (row & 7)) << 4)) = v;
          }
        }
        tc_fence_before();
        mbar_arrive(bar(B_OE + x));                // O_x has been read: the next item may overwrite it
        const int tt = m.t0 + x * p.TOK + row / p.G;
        if (tt < p.T && p.lse != nullptr)
          p.lse[((long long)m.b * p.Hq + m.h * p.G + g_in_row) * p.T + tt] =
              (m_ref + __log2f(l_sum)) * 0.69314718055994531f;
        fence_proxy_async();
        mbar_arrive(bar(B_STG + x));                // this row is staged (warp 2 + x stores it)
      }
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

}  // namespace tc

bool attn_prefill_tc_supported(const lte_dims* d) {
  const int G = d->Hq / d->Hkv;
  return d->dtype == LTE_BF16 && d->D == tc::HD &&
         (G == 1 || G == 2 || G == 4 || G == 8 || G == 16);
}

// Tensor maps need every byte stride a multiple of 16 (pointers are checked at the API).
bool attn_prefill_tc_layout_ok(const PrefillArgs& a) {
  const Strides4* ss[3] = {&a.qs, &a.kvs, &a.os};
  for (const Strides4* s : ss)
    if ((s->h * 2) % 16 != 0 || (s->t * 2) % 16 != 0 || (s->b * 2) % 16 != 0) return false;
  return true;
}

cudaError_t attn_prefill_tc(const PrefillArgs& a, cudaStream_t stream) {
  using namespace tc;
  const lte_dims* d = a.d;
  const int G = d->Hq / d->Hkv, TOK = BM / G;
  CUtensorMap mq, mk, mv, mkc, mvc, mo;
  {
    // Q rows are loaded and O rows stored in the same box: G heads x TOK tokens
    const cuuint64_t dims[4] = {(cuuint64_t)HD, (cuuint64_t)d->Hq, (cuuint64_t)d->T, (cuuint64_t)d->B};
    const cuuint64_t st[3] = {(cuuint64_t)a.qs.h * 2, (cuuint64_t)a.qs.t * 2, (cuuint64_t)a.qs.b * 2};
    const cuuint64_t so[3] = {(cuuint64_t)a.os.h * 2, (cuuint64_t)a.os.t * 2, (cuuint64_t)a.os.b * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)TOK, 1};
    if (!encode(&mq, a.q, 4, dims, st, box)) return cudaErrorInvalidValue;
    if (!encode(&mo, a.o, 4, dims, so, box)) return cudaErrorInvalidValue;
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
  p.sink = d->sink; p.window = d->window; p.cap = d->cap; p.cap_policy = d->cap_policy;
  p.n_pairs = (d->T + 2 * TOK - 1) / (2 * TOK);
  p.n_units = d->B * d->Hkv;
  p.n_items = p.n_pairs * p.n_units;
  p.scale_log2 = d->scale * 1.4426950408889634f;
  p.cnt = a.cnt;
  p.death = a.death;
  p.bias = a.bias;
  p.col_stride = d->sink + d->T;
  p.lse = a.lse; p.err = a.err;
  auto kernel = a.death != nullptr
                    ? (a.bias != nullptr ? attn_prefill_tc_kernel<true, true>
                                         : attn_prefill_tc_kernel<true, false>)
                    : (a.bias != nullptr ? attn_prefill_tc_kernel<false, true>
                                         : attn_prefill_tc_kernel<false, false>);
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, n_sm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  const int grid = p.n_items < n_sm ? p.n_items : n_sm;
  kernel<<<grid, kThreads, kSmemBytes, stream>>>(mq, mk, mv, mkc, mvc, mo, p);
  return cudaGetLastError();
}

}  // namespace lte
