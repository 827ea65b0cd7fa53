// CUDA-core compress / append kernel: z = x · A into the paged latent cache.
//
// Method: "PALU 论文低秩投影分解" §低秩投影分解 (z_k = x A_k, z_v = x A_v) and
// §把它放进一次真实推理流程里看, Prefill 阶段 (compute the latents and cache them).
// Each output row is accumulated in float32, rounded to nearest even into the
// latent dtype (or quantised to int4 with a per-32-entry fp16 scale) and
// scattered to its slot page·P + offset.
#include "palu_common.cuh"
#include "palu_internal.h"

namespace palu {
namespace {

constexpr int kBM = 64, kBN = 64, kBK = 32, kThreads = 256;

template <int ACT, int LAT>
__global__ void __launch_bounds__(kThreads) compress_kernel(const __grid_constant__ CompressArgs a) {
  using TA = typename Dt<ACT>::T;
  __shared__ float xs[kBK][kBM + 1];
  __shared__ float as_[kBK][kBN + 1];
  __shared__ float ct[kBM][kBN + 1];
  DevStatus* st = reinterpret_cast<DevStatus*>(a.status);

  const bool is_v = blockIdx.z == 1;
  // output column gc belongs to entry col_entry(cols, n, gc), latent entry gc - cols[entry]
  const uint16_t* cols = is_v ? a.vcol : a.kcol;
  const int N = is_v ? a.ncols_v : a.ncols_k;
  const long long acols = is_v ? a.a_vcols : a.a_kcols;
  const uint16_t* col0s = is_v ? a.gm.v_row0 : a.gm.k_row0;
  const int row0 = blockIdx.x * kBM, col0 = blockIdx.y * kBN;
  if (col0 >= N) return;
  const TA* X = reinterpret_cast<const TA*>(a.x);
  const TA* A = reinterpret_cast<const TA*>(is_v ? a.Av : a.Ak);
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;

  float acc[4][4] = {};
  for (int k0 = 0; k0 < a.d_model; k0 += kBK) {
    for (int e = tid; e < kBM * kBK; e += kThreads) {
      const int i = e / kBK, k = e % kBK;
      const int gi = row0 + i, gk = k0 + k;
      xs[k][i] = (gi < a.n && gk < a.d_model) ? Dt<ACT>::to_f(X[(size_t)gi * a.d_model + gk]) : 0.f;
    }
    for (int e = tid; e < kBK * kBN; e += kThreads) {
      const int k = e / kBN, c = e % kBN;
      const int gk = k0 + k, gc = col0 + c;
      float v = 0.f;
      if (gk < a.d_model && gc < N) {
        const int e = col_entry(cols, a.gm.n, gc);
        v = Dt<ACT>::to_f(A[(size_t)gk * acols + col0s[e] + (gc - cols[e])]);
      }
      as_[k][c] = v;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kBK; ++k) {
      float xv[4], av[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        xv[u] = xs[k][ty * 4 + u];
        av[u] = as_[k][tx * 4 + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(xv[u], av[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) ct[ty * 4 + u][tx * 4 + v] = acc[u][v];
  __syncthreads();

  const long long cap = (long long)a.num_pages * a.P;
  const long long page_bytes = is_v ? a.gm.v_page : a.gm.k_page;

  if constexpr (LAT == PALU_INT4) {
    // one thread per (token row, 32-entry block)
    const long long spage = is_v ? a.gm.vs_page : a.gm.ks_page;
    if (tid < kBM * 2) {
      const int i = tid / 2, blk = tid % 2;
      const int gi = row0 + i, gc = col0 + blk * 32;
      if (gi < a.n && gc < N) {
        const int slot = a.slots[gi];
        if (slot >= 0) {
          if (slot >= cap) {
            report(st, PALU_ERR_DEVICE_BOUNDS, 3000000 + gi);
          } else {
            const int e = col_entry(cols, a.gm.n, gc), j0 = gc - cols[e];
            const long long srow = int4_scale_row(cols[e + 1] - cols[e]);
            const int tok = slot % a.P;
            uint8_t* pblk = const_cast<uint8_t*>(is_v ? a.gm.zv[e] : a.gm.zk[e]) + (long long)(slot / a.P) * page_bytes;
            uint8_t* sblk = const_cast<uint8_t*>(is_v ? a.gm.zvs[e] : a.gm.zks[e]) + (long long)(slot / a.P) * spage;
            float amax = 0.f;
            for (int u = 0; u < 32; ++u) amax = fmaxf(amax, fabsf(ct[i][blk * 32 + u]));
            const __half s16 = __float2half_rn(__fdiv_rn(amax, 7.0f));
            const float s = __half2float(s16);
            uint32_t words[4] = {0, 0, 0, 0};
            for (int u = 0; u < 32; ++u) {
              int code = 0;
              if (s != 0.f) {
                float qv = rintf(__fdiv_rn(ct[i][blk * 32 + u], s));
                qv = fminf(fmaxf(qv, -7.f), 7.f);
                code = (int)qv;
              }
              words[u / 8] |= (uint32_t)(code & 0xF) << (4 * (u % 8));
            }
            // 32 codes = one 16-byte unit of the swizzled page block
            uint4* dst = reinterpret_cast<uint4*>(pblk + swz_offset(tok, j0 / 2, a.P));
            *dst = make_uint4(words[0], words[1], words[2], words[3]);
            reinterpret_cast<__half*>(sblk + tok * srow)[j0 / 32] = s16;
          }
        }
      }
    }
  } else {
    using TL = typename Dt<LAT>::T;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = ty * 4 + u, gi = row0 + i;
      if (gi >= a.n) continue;
      const int slot = a.slots[gi];
      if (slot < 0) continue;
      if (slot >= cap) {
        report(st, PALU_ERR_DEVICE_BOUNDS, 3000000 + gi);
        continue;
      }
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int gc = col0 + tx * 4 + v;
        if (gc >= N) continue;
        const int e = col_entry(cols, a.gm.n, gc), j = gc - cols[e];
        uint8_t* blk = const_cast<uint8_t*>(is_v ? a.gm.zv[e] : a.gm.zk[e]) + (long long)(slot / a.P) * page_bytes;
        *reinterpret_cast<TL*>(blk + swz_offset(slot % a.P, (long long)j * sizeof(TL), a.P)) =
            Dt<LAT>::from_f(ct[i][tx * 4 + v]);
      }
    }
  }

  // positions: once per token, by the first column tile of the key side
  if (blockIdx.y == 0 && !is_v && a.positions != nullptr && a.pos_pool != nullptr && tid < kBM) {
    const int gi = row0 + tid;
    if (gi < a.n) {
      const int slot = a.slots[gi];
      if (slot >= 0 && slot < cap) a.pos_pool[slot] = a.positions[gi];
    }
  }
}

template <int ACT, int LAT>
cudaError_t launch_t(const CompressArgs& a, cudaStream_t st) {
  const int ncol = a.ncols_k > a.ncols_v ? a.ncols_k : a.ncols_v;
  dim3 grid((a.n + kBM - 1) / kBM, (ncol + kBN - 1) / kBN, 2);
  compress_kernel<ACT, LAT><<<grid, kThreads, 0, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_compress_simt(const CompressArgs& a, cudaStream_t st) {
  if (a.act == PALU_F32 && a.lat == PALU_F32) return launch_t<PALU_F32, PALU_F32>(a, st);
  if (a.act == PALU_F16 && a.lat == PALU_F16) return launch_t<PALU_F16, PALU_F16>(a, st);
  if (a.act == PALU_BF16 && a.lat == PALU_BF16) return launch_t<PALU_BF16, PALU_BF16>(a, st);
  if (a.act == PALU_F16 && a.lat == PALU_INT4) return launch_t<PALU_F16, PALU_INT4>(a, st);
  if (a.act == PALU_BF16 && a.lat == PALU_INT4) return launch_t<PALU_BF16, PALU_INT4>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace palu
