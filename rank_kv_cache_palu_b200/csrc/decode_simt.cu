// CUDA-core decode kernels: the split kernel for float32 caches (and any shape
// the tensor-core kernel does not take), and the log-sum-exp combine that
// every decode path ends with.
//
// Method: "PALU 论文低秩投影分解" §低秩投影分解 (K ≈ z_k B_k, V ≈ z_v B_v) and
// §把它放进一次真实推理流程里看, Decode 阶段 (rebuild keys from the cached
// latents on the fly; keep values in latent space so V is never built).
#include <math.h>

#include "palu_common.cuh"
#include "palu_internal.h"

namespace palu {
namespace {

constexpr int kThreads = 128;
constexpr int kTT = 16;  // tokens per tile

// Per-sequence split bounds: the context is cut at page boundaries into S
// ranges of ceil(pages/S) pages each.
struct SplitRange {
  int t_begin, t_end;
};

__device__ __forceinline__ int checked_len(const DecodeArgs& a, int b, DevStatus* st) {
  int T = a.seq_lens[b];
  const int cap = a.max_pages * a.P;
  if (T < 0 || T > cap) {
    report(st, PALU_ERR_DEVICE_BOUNDS, 1000000 + b);
    T = T < 0 ? 0 : cap;
  }
  return T;
}

__device__ __forceinline__ SplitRange split_range(int T, int P, int S, int s) {
  const int npg = (T + P - 1) / P;
  const int pps = (npg + S - 1) / S;
  const int pg0 = s * pps;
  const int pg1 = min(npg, pg0 + pps);
  SplitRange r;
  r.t_begin = pg0 * P;
  r.t_end = min(T, pg1 * P);
  if (r.t_end < r.t_begin) r.t_end = r.t_begin;
  return r;
}

template <int ACT, int LAT>
__global__ void __launch_bounds__(kThreads) split_kernel(const __grid_constant__ DecodeArgs a) {
  using TA = typename Dt<ACT>::T;
  extern __shared__ float smem[];
  // blockIdx.y: head hl of this launch; entry i = hl / gs of the group map
  const int s = blockIdx.x, hl = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int gi = hl / a.gs, jh = hl % a.gs;
  const int h = a.gm.g[gi] * a.gs + jh;   // model head
  const int r_k = a.gm.rk[gi];            // this group's key rank (<= a.r_k)
  const long long ks_row = (2 * (r_k / 32) + 15) / 16 * 16;   // int4 scale row bytes of this group
  const int d_h = a.d_h, half = d_h / 2;
  DevStatus* st = reinterpret_cast<DevStatus*>(a.status);

  float* qr = smem;                       // [d_h] rotated, scaled query
  float* zk_t = qr + d_h;                 // [kTT][r_k]
  float* zv_t = zk_t + kTT * r_k;         // [kTT][r_v]
  float* kt = zv_t + kTT * a.r_v;         // [kTT][d_h]
  float* sc = kt + kTT * d_h;             // [kTT] scores
  int* tpos = reinterpret_cast<int*>(sc + kTT);  // [kTT] positions

  const int T = checked_len(a, b, st);
  const SplitRange rg = split_range(T, a.P, a.S, s);

  // Rotated query, with the softmax scale folded in.
  const TA* qh = reinterpret_cast<const TA*>(a.q) + (size_t)b * a.q_bstride + (size_t)h * d_h;
  const int qpos = a.q_pos[(size_t)b * a.qpos_bstride];
  for (int i = tid; i < half; i += kThreads) {
    const float x1 = Dt<ACT>::to_f(qh[i]), x2 = Dt<ACT>::to_f(qh[i + half]);
    float c = 1.f, sn = 0.f;
    if (a.rope) rope_cs_accurate(qpos, a.omega[i], c, sn);
    qr[i] = (x1 * c - x2 * sn) * a.sm_scale;
    qr[i + half] = (x2 * c + x1 * sn) * a.sm_scale;
  }

  constexpr int kMaxRv = 512;
  float acc_v[kMaxRv / kThreads];
#pragma unroll
  for (int k = 0; k < kMaxRv / kThreads; ++k) acc_v[k] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;

  const TA* Bk = reinterpret_cast<const TA*>(a.Bk) + (size_t)a.gm.k_row0[gi] * a.W + jh * d_h;
  const uint8_t* zk_base = a.gm.zk[gi];
  const uint8_t* zv_base = a.gm.zv[gi];
  const uint8_t* zks_base = a.gm.zks[gi];
  const uint8_t* zvs_base = a.gm.zvs[gi];
  const int32_t* ptab = a.page_table + (size_t)b * a.max_pages;

  for (int t0 = rg.t_begin; t0 < rg.t_end; t0 += kTT) {
    const int nt = min(kTT, rg.t_end - t0);
    __syncthreads();  // previous tile fully consumed
    // ---- stage the tile's latents as float
    if (tid < kTT) {
      int pv = 0;
      if (tid < nt) {
        const int t = t0 + tid;
        int page = ptab[t / a.P];
        if (page < 0 || page >= a.num_pages) page = -1;
        pv = (a.pos_pool != nullptr && page >= 0) ? a.pos_pool[(size_t)page * a.P + t % a.P] : t;
      }
      tpos[tid] = pv;
    }
    for (int e = tid; e < kTT * r_k; e += kThreads) {
      const int tt = e / r_k, j = e % r_k;
      float v = 0.f;
      if (tt < nt) {
        const int t = t0 + tt;
        const int page = ptab[t / a.P];
        if (page < 0 || page >= a.num_pages) {
          report(st, PALU_ERR_DEVICE_BOUNDS, 2000000 + b);
        } else {
          v = load_latent<LAT, ACT>(zk_base + (size_t)page * a.gm.k_page, t % a.P, a.P,
                                    LAT == PALU_INT4 ? zks_base + (size_t)page * a.gm.ks_page +
                                                           (size_t)(t % a.P) * ks_row
                                                     : nullptr,
                                    j);
        }
      }
      zk_t[e] = v;
    }
    for (int e = tid; e < kTT * a.r_v; e += kThreads) {
      const int tt = e / a.r_v, j = e % a.r_v;
      float v = 0.f;
      if (tt < nt) {
        const int t = t0 + tt;
        const int page = ptab[t / a.P];
        if (page >= 0 && page < a.num_pages) {
          v = load_latent<LAT, ACT>(zv_base + (size_t)page * a.gm.v_page, t % a.P, a.P,
                                    LAT == PALU_INT4 ? zvs_base + (size_t)page * a.gm.vs_page +
                                                           (size_t)(t % a.P) * a.vs_row
                                                     : nullptr,
                                    j);
        }
      }
      zv_t[e] = v;
    }
    __syncthreads();
    // ---- key reconstruction: kt[tt][d] = Σ_r zk[tt][r] · B_k[g][r][jh·d_h + d]
    for (int d = tid; d < d_h; d += kThreads) {
      float acc[kTT];
#pragma unroll
      for (int tt = 0; tt < kTT; ++tt) acc[tt] = 0.f;
      for (int r = 0; r < r_k; ++r) {
        const float bv = Dt<ACT>::to_f(Bk[(size_t)r * a.W + d]);
#pragma unroll
        for (int tt = 0; tt < kTT; ++tt) acc[tt] = fmaf(zk_t[tt * r_k + r], bv, acc[tt]);
      }
#pragma unroll
      for (int tt = 0; tt < kTT; ++tt) kt[tt * d_h + d] = acc[tt];
    }
    __syncthreads();
    // ---- RoPE on the keys and scores: 8 lanes per token
    {
      const int tt = tid >> 3, lane8 = tid & 7;
      float part = 0.f;
      if (tt < nt) {
        const int pv = tpos[tt];
        for (int i = lane8; i < half; i += 8) {
          const float k1 = kt[tt * d_h + i], k2 = kt[tt * d_h + i + half];
          float c = 1.f, sn = 0.f;
          if (a.rope) rope_cs_accurate(pv, a.omega[i], c, sn);
          part = fmaf(k1 * c - k2 * sn, qr[i], part);
          part = fmaf(k2 * c + k1 * sn, qr[i + half], part);
        }
      }
#pragma unroll
      for (int off = 4; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      if (lane8 == 0 && tt < kTT) sc[tt] = (tt < nt && (!a.causal || tpos[tt] <= qpos)) ? part : -INFINITY;
    }
    __syncthreads();
    // ---- online softmax and the latent value sum
    float m_tile = -INFINITY;
    for (int tt = 0; tt < nt; ++tt) m_tile = fmaxf(m_tile, sc[tt]);
    const float m_new = fmaxf(m_run, m_tile);
    const float resc = (m_run == -INFINITY) ? 0.f : expf(m_run - m_new);
    float psum = 0.f;
    float p[kTT];
#pragma unroll
    for (int tt = 0; tt < kTT; ++tt) {
      p[tt] = (tt < nt && m_new != -INFINITY) ? expf(sc[tt] - m_new) : 0.f;   // all masked so far: nothing
      psum += p[tt];
    }
    l_run = l_run * resc + psum;
    m_run = m_new;
#pragma unroll
    for (int k = 0; k < kMaxRv / kThreads; ++k) {
      const int r = tid + k * kThreads;
      if (r < a.r_v) {
        float v = acc_v[k] * resc;
#pragma unroll
        for (int tt = 0; tt < kTT; ++tt) v = fmaf(p[tt], zv_t[tt * a.r_v + r], v);
        acc_v[k] = v;
      }
    }
  }

  float* out = a.part + (((size_t)b * a.gm.n * a.gs + hl) * a.S + s) * (a.r_v + 2);
  if (tid == 0) {
    out[0] = m_run;
    out[1] = l_run;
  }
#pragma unroll
  for (int k = 0; k < kMaxRv / kThreads; ++k) {
    const int r = tid + k * kThreads;
    if (r < a.r_v) out[2 + r] = acc_v[k];
  }
}

// Log-sum-exp merge of the split partials, then the value up-projection
// out_h = a_h · B_v[g][:, cols_h] (a GEMV per (sequence, head)): 256 threads =
// 64 output pairs × 4 interleaved quarters of the latent rows, two accumulator
// chains each, summed across the quarters in shared memory.
template <typename TA>
struct Pair;
template <> struct Pair<float> {
  __device__ __forceinline__ static float2 load(const float* p) { return *reinterpret_cast<const float2*>(p); }
};
template <> struct Pair<__half> {
  __device__ __forceinline__ static float2 load(const __half* p) {
    return __half22float2(*reinterpret_cast<const __half2*>(p));
  }
};
template <> struct Pair<__nv_bfloat16> {
  __device__ __forceinline__ static float2 load(const __nv_bfloat16* p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
  }
};

constexpr int kCombineThreads = 256;   // 64 output pairs x 4 row quarters

template <int ACT>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const __grid_constant__ DecodeArgs a) {
  using TA = typename Dt<ACT>::T;
  constexpr int kThreads = kCombineThreads;
  extern __shared__ float smem[];
  float* av = smem;             // [r_v]
  float* wgt = av + a.r_v;      // [S]
  float* red = wgt + a.S;       // [4][d_h] per-quarter outputs
  // blockIdx.x: head hl of this launch (entry hl / gs of the group map)
  const int hl = blockIdx.x, vb = blockIdx.y;
  const int b = vb / a.qn, jq = vb % a.qn;
  const int tid = threadIdx.x;
  const int gi = hl / a.gs, jh = hl % a.gs;
  const int h = a.gm.g[gi] * a.gs + jh;   // model head
  const float* part = a.part + ((size_t)vb * a.gm.n * a.gs + hl) * a.S * (a.r_v + 2);

  float M = -INFINITY;
  for (int s = 0; s < a.S; ++s) M = fmaxf(M, part[(size_t)s * (a.r_v + 2)]);
  TA* out = reinterpret_cast<TA*>(a.out) + (size_t)b * a.o_bstride + ((size_t)jq * a.H + h) * a.d_h;
  if (M == -INFINITY) {
    for (int d = tid; d < a.d_h; d += kThreads) out[d] = Dt<ACT>::from_f(0.f);
    if (tid == 0 && a.lse != nullptr) a.lse[(size_t)b * a.lse_bstride + (size_t)jq * a.H + h] = -INFINITY;
    return;
  }
  float L = 0.f;
  for (int s = 0; s < a.S; ++s) {
    const float ms = part[(size_t)s * (a.r_v + 2)];
    const float w = (ms == -INFINITY) ? 0.f : expf(ms - M);
    L += w * part[(size_t)s * (a.r_v + 2) + 1];
    if (tid == 0) wgt[s] = w;
  }
  __syncthreads();
  const float invL = 1.f / L;
  for (int r = tid; r < a.r_v; r += kThreads) {
    float v = 0.f;
    for (int s = 0; s < a.S; ++s) {
      const float w = wgt[s];
      if (w != 0.f) v = fmaf(w, part[(size_t)s * (a.r_v + 2) + 2 + r], v);
    }
    av[r] = v * invL;
  }
  __syncthreads();
  const TA* Bv = reinterpret_cast<const TA*>(a.Bv) + (size_t)a.gm.v_row0[gi] * a.W + jh * a.d_h;
  const int dp = tid & 63, rq = tid >> 6;
  const int d0 = 2 * dp;
  if (d0 < a.d_h) {
    float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0;
    int r = rq;
    for (; r + 4 < a.r_v; r += 8) {
      const float2 b0 = Pair<TA>::load(Bv + (size_t)r * a.W + d0);
      const float2 b1 = Pair<TA>::load(Bv + (size_t)(r + 4) * a.W + d0);
      acc0.x = fmaf(av[r], b0.x, acc0.x);
      acc0.y = fmaf(av[r], b0.y, acc0.y);
      acc1.x = fmaf(av[r + 4], b1.x, acc1.x);
      acc1.y = fmaf(av[r + 4], b1.y, acc1.y);
    }
    if (r < a.r_v) {
      const float2 b0 = Pair<TA>::load(Bv + (size_t)r * a.W + d0);
      acc0.x = fmaf(av[r], b0.x, acc0.x);
      acc0.y = fmaf(av[r], b0.y, acc0.y);
    }
    red[rq * a.d_h + d0] = acc0.x + acc1.x;
    red[rq * a.d_h + d0 + 1] = acc0.y + acc1.y;
  }
  __syncthreads();
  for (int d = tid; d < a.d_h; d += kThreads) {
    const float o = (red[d] + red[a.d_h + d]) + (red[2 * a.d_h + d] + red[3 * a.d_h + d]);
    out[d] = Dt<ACT>::from_f(o);
  }
  if (tid == 0 && a.lse != nullptr) a.lse[(size_t)b * a.lse_bstride + (size_t)jq * a.H + h] = M + logf(L);
}

template <int ACT, int LAT>
cudaError_t launch_split_t(const DecodeArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(float) * (a.d_h + kTT * (a.r_k + a.r_v + a.d_h) + kTT) + sizeof(int) * kTT;
  auto kern = split_kernel<ACT, LAT>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(a.S, a.gm.n * a.gs, a.batch);
  kern<<<grid, kThreads, smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t st) {
  if (a.act == PALU_F32 && a.lat == PALU_F32) return launch_split_t<PALU_F32, PALU_F32>(a, st);
  if (a.act == PALU_F16 && a.lat == PALU_F16) return launch_split_t<PALU_F16, PALU_F16>(a, st);
  if (a.act == PALU_BF16 && a.lat == PALU_BF16) return launch_split_t<PALU_BF16, PALU_BF16>(a, st);
  if (a.act == PALU_F16 && a.lat == PALU_INT4) return launch_split_t<PALU_F16, PALU_INT4>(a, st);
  if (a.act == PALU_BF16 && a.lat == PALU_INT4) return launch_split_t<PALU_BF16, PALU_INT4>(a, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(float) * (a.r_v + a.S + 4 * a.d_h);
  dim3 grid(a.gm.n * a.gs, a.batch * a.qn);
  if (a.act == PALU_F32) combine_kernel<PALU_F32><<<grid, kCombineThreads, smem, st>>>(a);
  else if (a.act == PALU_F16) combine_kernel<PALU_F16><<<grid, kCombineThreads, smem, st>>>(a);
  else if (a.act == PALU_BF16) combine_kernel<PALU_BF16><<<grid, kCombineThreads, smem, st>>>(a);
  else return cudaErrorInvalidValue;
  count_launch();
  return cudaGetLastError();
}

}  // namespace palu
