// Decode step of LTE: cache update, deferred batched scoring, split-KV
// attention with an in-kernel log-sum-exp merge.
//
// "Alleviating Forgetfulness of Linear Attention by Hybrid Sparse Attention
// and Contextualized Learnable Token Eviction", Fig. 3 caption: the inference
// cache is a circular segment for in-window KVs plus an out-of-window segment
// of capped capacity for the retained KVs and the attention sink; scoring is
// batched and deferred as late as possible.  Fig. 2 caption: a KV pair is
// kept or evicted when it moves out of the window.  "Sparse Linear Attention:
// Viewing SWA from the Perspective of Linear Attention", section "Viewing SWA
// from the linear-state perspective": each new token overwrites one slot of
// the window (FIFO).
//
// Per step (all kernels read the step index t from meta[0] on the device, so
// the same launches replay unchanged inside a CUDA graph):
//  1. decode_update_kernel (one CTA per (batch, KV head) unit): token t-w
//     leaves its window slot (sink slot, retained ring, or dropped); token t
//     takes slot t mod w.
//  2. score_ring (score_cnn.cu): when score_batch tokens are scorable, score
//     them from the window segment.
//  3. decode_attn_kernel: the unit's valid slots (window, sinks, retained) are
//     one logical key list split into chunks of 128 keys, one CTA per chunk;
//     four warps stream 32 keys each through shared memory with cp.async and
//     run QK^T and PV on m16n8k16 bf16 MMAs (the G query heads of the group
//     are rows of the A operand, so each K/V byte is read once per group).
//     Each CTA writes an (m, l, o) partial; the last CTA of a unit (atomic
//     counter) merges them; the last unit advances meta.
#include <math.h>

#include <mutex>

#include "lte_common.cuh"
#include "lte_internal.h"

namespace lte {

constexpr int kDecKeysPerWarp = 32;
constexpr int kDecWarps = 4;
constexpr int kDecKeysPerCta = kDecKeysPerWarp * kDecWarps;
constexpr int kDecThreads = 32 * kDecWarps;

static inline int dec_splits(const lte_dims* d) {
  const int L = d->window + d->sink + d->cap;
  return (L + kDecKeysPerCta - 1) / kDecKeysPerCta;
}

// workspace layout after the error word: partials [units][splits][G][D+2] fp32,
// then counters [units + 1] int32.
size_t decode_scratch_bytes(const lte_dims* d) {
  const size_t units = (size_t)d->B * d->Hkv;
  const size_t G = d->Hq / d->Hkv;
  return units * dec_splits(d) * G * (d->D + 2) * sizeof(float) + (units + 1) * sizeof(int32_t) +
         64;
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
decode_update_kernel(int Hkv, int D, int elt, int window, int sink, int cap, float tau,
                     const char* __restrict__ k_t, const char* __restrict__ v_t,
                     char* __restrict__ ck, char* __restrict__ cv, int32_t* __restrict__ pos,
                     float* __restrict__ win_r, int32_t* __restrict__ ret_total,
                     const int32_t* __restrict__ meta, int32_t* __restrict__ counters,
                     int n_units, DevError* err) {
  const int u = blockIdx.x, tid = threadIdx.x;
  const int L = window + sink + cap;
  const int t = meta[0];
  const int leaving = t - window;
  const int slot_w = t % window;
  const long long urow = (long long)u * L;
  int dst_slot = -1, rt = 0;
  bool retained = false;
  if (leaving >= 0) {
    if (pos[urow + slot_w] != leaving) {
      if (tid == 0) record_error(err, LTE_ERR_DEVICE, kWhereDecodeIndex);
    } else if (leaving < sink) {
      dst_slot = window + leaving;
    } else if (cap > 0 && win_r[(long long)u * window + slot_w] >= tau) {
      rt = ret_total[u];
      dst_slot = window + sink + rt % cap;
      retained = true;
    }
  }
  const int nvec = D * elt / 16;
  const long long wsrc = (urow + slot_w) * D * elt;
  for (int i = tid; i < nvec; i += blockDim.x) {
    uint4* kw = reinterpret_cast<uint4*>(ck + wsrc) + i;
    uint4* vw = reinterpret_cast<uint4*>(cv + wsrc) + i;
    if (dst_slot >= 0) {
      const long long dst = (urow + dst_slot) * D * elt;
      reinterpret_cast<uint4*>(ck + dst)[i] = *kw;
      reinterpret_cast<uint4*>(cv + dst)[i] = *vw;
    }
    *kw = reinterpret_cast<const uint4*>(k_t + (long long)u * D * elt)[i];
    *vw = reinterpret_cast<const uint4*>(v_t + (long long)u * D * elt)[i];
  }
  if (tid == 0) {
    if (dst_slot >= 0) pos[urow + dst_slot] = leaving;
    if (retained) ret_total[u] = rt + 1;
    pos[urow + slot_w] = t;
    win_r[(long long)u * window + slot_w] = NAN;
    counters[u] = 0;
    if (u == 0) counters[n_units] = 0;
  }
}

// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32d(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16d(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void ldsm_x4d(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                         uint32_t& r3, bool trans) {
  if (trans)
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
  else
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16d(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16d(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
template <int D>
__device__ __forceinline__ uint32_t swzd(int r, int c) {
  return (uint32_t)(r * D * 2 + ((c ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kDecThreads)
decode_attn_kernel(int Hq, int Hkv, int window, int sink, int cap, float scale_log2,
                   const __nv_bfloat16* __restrict__ q_t, const __nv_bfloat16* __restrict__ ck,
                   const __nv_bfloat16* __restrict__ cv, const int32_t* __restrict__ ret_total,
                   int32_t* __restrict__ meta, __nv_bfloat16* __restrict__ o_t,
                   float* __restrict__ lse_t, float* __restrict__ part,
                   int32_t* __restrict__ counters, int n_units, int n_split) {
  constexpr int CH = D / 8, KSTEPS = D / 16, DN = D / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* q_sm = smem;                                   // [16][D] bf16
  uint8_t* kv_sm = smem + 16 * D * 2;                     // per warp: K [32][D], V [32][D]
  __shared__ float m_sh[kDecWarps][16], l_sh[kDecWarps][16];
  __shared__ int is_last;

  const int split = blockIdx.x, u = blockIdx.y;
  const int b = u / Hkv, h = u % Hkv, G = Hq / Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L = window + sink + cap;
  const int t = meta[0];
  const int nw = min(window, t + 1);
  int ns = t - window + 1;
  ns = ns < 0 ? 0 : (ns > sink ? sink : ns);
  const int rt = ret_total[u];
  const int nr = min(cap, rt);
  const int n = nw + ns + nr;

  // Q rows 0..G-1 (rows G..15 zero)
  for (int i = tid; i < 16 * CH; i += kDecThreads) {
    const int r = i / CH, c = i % CH;
    const bool ok = r < G;
    const __nv_bfloat16* src = q_t + (ok ? ((long long)b * Hq + h * G + r) * D + c * 8 : 0);
    cp_async16d(smem_u32d(q_sm + swzd<D>(r, c)), src, ok);
  }
  // this warp's 32 keys: logical l -> slot
  const int l0 = split * kDecKeysPerCta + warp * kDecKeysPerWarp;
  uint8_t* ks = kv_sm + warp * 2 * kDecKeysPerWarp * D * 2;
  uint8_t* vs = ks + kDecKeysPerWarp * D * 2;
  const long long ubase = (long long)u * L;
  for (int i = lane; i < kDecKeysPerWarp * CH; i += 32) {
    const int r = i / CH, c = i % CH;
    const int l = l0 + r;
    const bool ok = l < n;
    int slot = 0;
    if (ok) slot = l < nw ? l : (l < nw + ns ? window + (l - nw) : window + sink + (l - nw - ns));
    const long long a = ok ? (ubase + slot) * D + c * 8 : 0;
    cp_async16d(smem_u32d(ks + swzd<D>(r, c)), ck + a, ok);
    cp_async16d(smem_u32d(vs + swzd<D>(r, c)), cv + a, ok);
  }
  asm volatile("cp.async.commit_group;\n" ::);
  asm volatile("cp.async.wait_group 0;\n" ::);
  __syncthreads();

  uint32_t qf[KSTEPS][4];
#pragma unroll
  for (int kst = 0; kst < KSTEPS; ++kst) {
    const int r = lane & 15, c = kst * 2 + (lane >> 4);
    ldsm_x4d(smem_u32d(q_sm + swzd<D>(r, c)), qf[kst][0], qf[kst][1], qf[kst][2], qf[kst][3],
             false);
  }
  float s[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
  for (int kst = 0; kst < KSTEPS; ++kst) {
#pragma unroll
    for (int np = 0; np < 2; ++np) {
      const int r = np * 16 + ((lane >> 4) << 3) + (lane & 7);
      const int c = kst * 2 + ((lane >> 3) & 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4d(smem_u32d(ks + swzd<D>(r, c)), b0, b1, b2, b3, false);
      mma_bf16d(s[2 * np], qf[kst], b0, b1);
      mma_bf16d(s[2 * np + 1], qf[kst], b2, b3);
    }
  }
  // mask keys beyond the list, softmax (exp2 domain)
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int l = l0 + nt * 8 + ((lane & 3) << 1) + (e & 1);
      s[nt][e] = (l < n) ? s[nt][e] * scale_log2 : -INFINITY;
      mx[e >> 1] = fmaxf(mx[e >> 1], s[nt][e]);
    }
  float m_use[2], l_part[2] = {0.f, 0.f};
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 1));
    mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 2));
    m_use[hr] = (mx[hr] == -INFINITY) ? 0.f : mx[hr];
  }
  uint32_t pf[2][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      p[e] = exp2f(s[nt][e] - m_use[e >> 1]);
      l_part[e >> 1] += p[e];
    }
    pf[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16d(p[0], p[1]);
    pf[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16d(p[2], p[3]);
  }
  float o_acc[DN][4];
#pragma unroll
  for (int i = 0; i < DN; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) o_acc[i][e] = 0.f;
#pragma unroll
  for (int kst = 0; kst < 2; ++kst) {
#pragma unroll
    for (int dp = 0; dp < DN / 2; ++dp) {
      const int r = kst * 16 + (((lane >> 3) & 1) << 3) + (lane & 7);
      const int c = dp * 2 + (lane >> 4);
      uint32_t b0, b1, b2, b3;
      ldsm_x4d(smem_u32d(vs + swzd<D>(r, c)), b0, b1, b2, b3, true);
      mma_bf16d(o_acc[2 * dp], pf[kst], b0, b1);
      mma_bf16d(o_acc[2 * dp + 1], pf[kst], b2, b3);
    }
  }
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    l_part[hr] += __shfl_xor_sync(0xffffffffu, l_part[hr], 1);
    l_part[hr] += __shfl_xor_sync(0xffffffffu, l_part[hr], 2);
  }
  // ---- merge the 4 warps through shared memory (reuses the K/V area)
  __syncthreads();
  float* o_sh = reinterpret_cast<float*>(kv_sm);          // [warps][16][D]
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int r = (lane >> 2) + hr * 8;
    if ((lane & 3) == 0) {
      m_sh[warp][r] = mx[hr];                             // -inf when the warp saw no key
      l_sh[warp][r] = l_part[hr];
    }
#pragma unroll
    for (int i = 0; i < DN; ++i) {
      const int dcol = i * 8 + ((lane & 3) << 1);
      o_sh[(warp * 16 + r) * D + dcol] = o_acc[i][hr * 2];
      o_sh[(warp * 16 + r) * D + dcol + 1] = o_acc[i][hr * 2 + 1];
    }
  }
  __syncthreads();
  // CTA partial for rows g < G:  part[u][split][g] = {m, l, o[D]}
  float* my_part = part + ((long long)u * n_split + split) * G * (D + 2);
  for (int i = tid; i < G * D; i += kDecThreads) {
    const int g = i / D, dd = i % D;
    float M = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, m_sh[w][g]);
    float acc = 0.f;
    for (int w = 0; w < kDecWarps; ++w)
      if (m_sh[w][g] != -INFINITY) acc += o_sh[(w * 16 + g) * D + dd] * exp2f(m_sh[w][g] - M);
    my_part[g * (D + 2) + 2 + dd] = acc;
    if (dd == 0) {
      float l = 0.f;
      for (int w = 0; w < kDecWarps; ++w)
        if (m_sh[w][g] != -INFINITY) l += l_sh[w][g] * exp2f(m_sh[w][g] - M);
      my_part[g * (D + 2)] = M;
      my_part[g * (D + 2) + 1] = l;
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = (atomicAdd(&counters[u], 1) == n_split - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // ---- last CTA of the unit: merge the splits
  const float* up = part + (long long)u * n_split * G * (D + 2);
  for (int i = tid; i < G * D; i += kDecThreads) {
    const int g = i / D, dd = i % D;
    float M = -INFINITY;
    for (int sp = 0; sp < n_split; ++sp) M = fmaxf(M, __ldcg(up + (sp * G + g) * (D + 2)));
    float acc = 0.f, l = 0.f;
    for (int sp = 0; sp < n_split; ++sp) {
      const float* pp = up + (sp * G + g) * (D + 2);
      const float m = __ldcg(pp);
      if (m == -INFINITY) continue;
      const float f = exp2f(m - M);
      l += __ldcg(pp + 1) * f;
      acc += __ldcg(pp + 2 + dd) * f;
    }
    o_t[((long long)b * Hq + h * G + g) * D + dd] = __float2bfloat16_rn(acc / l);
    if (dd == 0 && lse_t != nullptr)
      lse_t[(long long)b * Hq + h * G + g] = (M + log2f(l)) * 0.69314718055994531f;
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(&counters[n_units], 1) == n_units - 1) {
      meta[0] = t + 1;
      meta[1] = meta[2];
    }
  }
}

template <int D>
static cudaError_t launch_decode_attn(const lte_dims* d, const lte_cache* c, const void* q_t,
                                      void* o_t, float* lse_t, float* part, int32_t* counters,
                                      cudaStream_t stream) {
  const int n_split = dec_splits(d);
  const int n_units = d->B * d->Hkv;
  const size_t smem = 16 * D * 2 + (size_t)kDecWarps * 2 * kDecKeysPerWarp * D * 2;
  cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(n_split, n_units);
  decode_attn_kernel<D><<<grid, kDecThreads, smem, stream>>>(
      d->Hq, d->Hkv, d->window, d->sink, d->cap, d->scale * 1.4426950408889634f,
      (const __nv_bfloat16*)q_t, (const __nv_bfloat16*)c->k, (const __nv_bfloat16*)c->v,
      c->ret_total, c->meta, (__nv_bfloat16*)o_t, lse_t, part, counters, n_units, n_split);
  return cudaGetLastError();
}

cudaError_t decode_step(const lte_dims* d, const lte_cnn* cnn, const lte_cache* c,
                        const void* q_t, const void* k_t, const void* v_t, void* o_t,
                        float* lse_t, int score_batch, DevError* err, void* scratch,
                        cudaStream_t stream) {
  const int n_units = d->B * d->Hkv;
  const int G = d->Hq / d->Hkv;
  float* part = reinterpret_cast<float*>(scratch);
  int32_t* counters = reinterpret_cast<int32_t*>(
      reinterpret_cast<char*>(scratch) +
      (size_t)n_units * dec_splits(d) * G * (d->D + 2) * sizeof(float));
  decode_update_kernel<<<n_units, 128, 0, stream>>>(
      d->Hkv, d->D, 2, d->window, d->sink, d->cap, d->tau, (const char*)k_t, (const char*)v_t,
      (char*)c->k, (char*)c->v, c->pos, c->win_r, c->ret_total, c->meta, counters, n_units, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = score_ring(d, cnn, c, score_batch, stream);
  if (e != cudaSuccess) return e;
  if (d->D == 128)
    return launch_decode_attn<128>(d, c, q_t, o_t, lse_t, part, counters, stream);
  return launch_decode_attn<64>(d, c, q_t, o_t, lse_t, part, counters, stream);
}

// ---------------------------------------------------------------------------
// Scratch of lte_decode_step_noalloc, for callers that cannot allocate device
// memory: one file-scope array per device, zero at module load, held until the
// process exits.  Host code must not pass the symbol itself to a kernel (on
// the host it names a stand-in, not device memory): the device address is
// looked up once per device with that device current, and cached.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LTE_NOALLOC_SCRATCH_BYTES];

cudaError_t noalloc_scratch(void** ptr) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  return cudaSuccess;
}

}  // namespace lte
