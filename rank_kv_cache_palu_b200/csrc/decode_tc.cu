// Tensor-core split kernel of the decode step (sm_100a: TMA + tcgen05 + TMEM).
//
// Method: "PALU 论文低秩投影分解" §低秩投影分解 (K ≈ z_k B_k, V ≈ z_v B_v) and
// §把它放进一次真实推理流程里看, Decode 阶段: keys are rebuilt from the cached
// latents tile by tile and never written out; values stay in latent space.
// "Palu: Compressing KV-Cache with Low-Rank Projection" (v2 abstract): the
// speed-ups are on RoPE-based attention, so every rebuilt key is rotated at its
// own position.
//
// One CTA = (sequence b, group g, head pair hp, split s); it walks the split's
// pages, 128 tokens (one page) per tile:
//   warp 0  TMA producer: B_k for the two heads once (MN-major, 128-byte
//           swizzle, resident), then the z_k page in 64-wide K chunks.
//   warp 6  TMA producer for z_v (its own ring, so neither stream waits on the other).
//   warp 1  MMA issuer: D[128 tok × 256] = z_k · B_k[:, 2 heads] into one of two
//           TMEM slots (kind::f16, fp32 accumulate); then aᵀ[r_v × 16] =
//           z_vᵀ · Pᵀ for the previous tile into the drained slot.
//   warps 2-5 epilogue, one thread per token: tcgen05.ld the rebuilt keys,
//           rotate them (RoPE at the token's position), score against the
//           rotated query, online softmax (exp2), write P (bf16/fp16) for the
//           value MMA, and fold each tile's aᵀ into running latent sums.
// Output: per (b, head, split) the partial (m, l, a[r_v]) the combine merges.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "palu_common.cuh"
#include "palu_internal.h"
#include "palu_tc.h"
#include "tc_ptx.cuh"

namespace palu {
namespace {

using namespace tc;

constexpr int kTile = 128;         // tokens per tile = page size
constexpr int kChunk = 64;         // K chunk of z_k (elements)
constexpr int kNKS = 3;            // z_k ring stages
constexpr int kNVS = 2;            // z_v ring stages
constexpr int kThreads = 224;      // 7 warps
constexpr int kZkBytes = kTile * kChunk * 2;   // 16 KB
constexpr int kZvBytes = 64 * 128 * 2;         // 16 KB: 64 tokens × 128 latent entries
constexpr int kPBytes = 16 * kTile * 2;        // 4 KB: 16 rows (heads, padded) × 128 tokens

struct Smem {
  // offsets in bytes from a 1024-aligned base
  uint32_t b, zk, zv, p, qr, omega, red, lred, bars, tmem_slot, abort, total;
};

__host__ __device__ inline Smem smem_layout(int r_k) {
  Smem s{};
  uint32_t o = 0;
  s.b = o;      o += (uint32_t)r_k * 256 * 2;          // B_k for 2 heads
  s.zk = o;     o += kNKS * kZkBytes;
  s.zv = o;     o += kNVS * kZvBytes;
  s.p = o;      o += 2 * kPBytes;
  s.qr = o;     o += 2 * 128 * 4;
  s.omega = o;  o += 64 * 8;
  s.red = o;    o += 2 * 4 * 2 * 4;
  s.lred = o;   o += 4 * 2 * 4;
  s.bars = o;   o += 32 * 8;
  s.tmem_slot = o; o += 16;
  s.abort = o;  o += 16;
  s.total = o;
  return s;
}

// barrier indices
enum {
  BAR_B = 0,
  BAR_ZK_FULL = 1,                   // kNKS
  BAR_ZK_EMPTY = BAR_ZK_FULL + kNKS,
  BAR_ZV_FULL = BAR_ZK_EMPTY + kNKS,  // kNVS
  BAR_ZV_EMPTY = BAR_ZV_FULL + kNVS,
  BAR_D_FULL = BAR_ZV_EMPTY + kNVS,  // 2
  BAR_D_EMPTY = BAR_D_FULL + 2,      // 2
  BAR_P_FULL = BAR_D_EMPTY + 2,      // 2
  BAR_AT_FULL = BAR_P_FULL + 2,      // 1
  BAR_TEARDOWN = BAR_AT_FULL + 1,
  BAR_EPI = BAR_TEARDOWN + 1,        // epilogue-wide sync (128 threads), bounded
  BAR_COUNT
};
static_assert(BAR_COUNT <= 32, "barrier space");

struct TileRange {
  int t_begin, t_end, ntiles;
  bool ragged_last;  // last tile shorter than a page: its value sum runs on CUDA cores
};

__device__ __forceinline__ TileRange tile_range(const DecodeArgs& a, int b, DevStatus* st, bool report_ok) {
  int T = a.seq_lens[b];
  const int cap = a.max_pages * a.P;
  if (T < 0 || T > cap) {
    if (report_ok) report(st, PALU_ERR_DEVICE_BOUNDS, 1000000 + b);
    T = T < 0 ? 0 : cap;
  }
  const int npg = (T + a.P - 1) / a.P;
  const int pps = (npg + a.S - 1) / a.S;
  const int s = blockIdx.x;
  const int pg0 = s * pps;
  const int pg1 = min(npg, pg0 + pps);
  TileRange r;
  r.t_begin = pg0 * a.P;
  r.t_end = max(r.t_begin, min(T, pg1 * a.P));
  r.ntiles = max(0, pg1 - pg0);
  r.ragged_last = r.ntiles > 0 && (r.t_end - (r.t_begin + (r.ntiles - 1) * kTile)) < kTile;
  return r;
}

// Physical page of logical page `lp`; -1 if the table entry is outside the pool.
__device__ __forceinline__ int page_of(const DecodeArgs& a, int b, int lp) {
  const int pg = a.page_table[(size_t)b * a.max_pages + lp];
  return (pg < 0 || pg >= a.num_pages) ? -1 : pg;
}

// P (softmax weights) tile, K-major with the 128-byte swizzle: row n (head),
// token k.  Tokens 0-63 and 64-127 sit in two 2 KB atoms of 16 rows.
__device__ __forceinline__ uint32_t p_offset(int n, int k) {
  const int region = k >> 6, kin = k & 63;
  const int chunk = (kin >> 3) ^ (n & 7);
  return (uint32_t)(region * 2048 + n * 128 + chunk * 16 + (kin & 7) * 2);
}

template <int ACT>
__device__ __forceinline__ uint16_t to_bits(float v) {
  if constexpr (ACT == PALU_BF16) {
    __nv_bfloat16 h = __float2bfloat16_rn(v);
    return *reinterpret_cast<uint16_t*>(&h);
  } else {
    __half h = __float2half_rn(v);
    return *reinterpret_cast<uint16_t*>(&h);
  }
}
template <int ACT>
__device__ __forceinline__ float from_bits(uint16_t u) {
  if constexpr (ACT == PALU_BF16) {
    return __bfloat162float(*reinterpret_cast<__nv_bfloat16*>(&u));
  } else {
    return __half2float(*reinterpret_cast<__half*>(&u));
  }
}

template <int ACT, int NRV>
__global__ void __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_zk, const __grid_constant__ CUtensorMap tm_zv,
                     const __grid_constant__ CUtensorMap tm_bk, const DecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  const Smem L = smem_layout(a.r_k);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  DevStatus* st = reinterpret_cast<DevStatus*>(a.status);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + L.abort);
  auto bar = [&](int i) { return base + L.bars + 8u * i; };

  const int b = blockIdx.z;
  const int nhp = a.gs / 2;                         // head pairs per group
  const int g = blockIdx.y / nhp, hp = blockIdx.y % nhp;
  const int nkc = a.r_k / kChunk;
  const int rows_total = a.num_pages * a.G * a.P;   // OOB row for bad pages => zero fill
  const TileRange tr = tile_range(a, b, st, threadIdx.x == 0);

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(BAR_B), 1);
    for (int i = 0; i < kNKS; ++i) {
      mbar_init(bar(BAR_ZK_FULL + i), 1);
      mbar_init(bar(BAR_ZK_EMPTY + i), 1);
    }
    for (int i = 0; i < kNVS; ++i) {
      mbar_init(bar(BAR_ZV_FULL + i), 1);
      mbar_init(bar(BAR_ZV_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(BAR_D_FULL + i), 1);
      mbar_init(bar(BAR_D_EMPTY + i), 4);
      mbar_init(bar(BAR_P_FULL + i), 4);
    }
    mbar_init(bar(BAR_AT_FULL), 1);
    mbar_init(bar(BAR_TEARDOWN), 1);
    mbar_init(bar(BAR_EPI), 128);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_zk);
    prefetch_tmap(&tm_zv);
    prefetch_tmap(&tm_bk);
  }
  if (warp == 1) {
    tmem_alloc(base + L.tmem_slot, 512);
    tmem_relinquish();
  }
  // zero the P buffers (padding rows stay zero), stage omega
  for (int i = threadIdx.x; i < 2 * kPBytes / 4; i += kThreads)
    reinterpret_cast<uint32_t*>(sbase + L.p)[i] = 0u;
  for (int i = threadIdx.x; i < 64; i += kThreads)
    reinterpret_cast<uint64_t*>(sbase + L.omega)[i] = a.omega[i];
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sbase + L.tmem_slot);

  if (warp == 0) {
    // ============================================================ z_k producer
    if (lane == 0) {
      mbar_expect_tx(bar(BAR_B), (uint32_t)a.r_k * 256 * 2);
      for (int nb = 0; nb < 4; ++nb)
        tma_load_2d(base + L.b + (uint32_t)nb * a.r_k * 128, &tm_bk, hp * 256 + nb * 64, g * a.r_k, bar(BAR_B));
      int stage = 0;
      uint32_t phase = 0;
      for (int k = 0; k < tr.ntiles && !*abort_flag; ++k) {
        const int lp = tr.t_begin / kTile + k;
        const int pg = page_of(a, b, lp);
        if (pg < 0) report(st, PALU_ERR_DEVICE_BOUNDS, 2000000 + b);
        const int row0 = pg < 0 ? rows_total : (pg * a.G + g) * a.P;
        for (int c = 0; c < nkc; ++c) {
          if (!mbar_wait(bar(BAR_ZK_EMPTY + stage), phase ^ 1, abort_flag, st, 10)) break;
          mbar_expect_tx(bar(BAR_ZK_FULL + stage), kZkBytes);
          tma_load_2d(base + L.zk + stage * kZkBytes, &tm_zk, c * kChunk, row0, bar(BAR_ZK_FULL + stage));
          if (++stage == kNKS) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 6) {
    // ============================================================ z_v producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int k = 0; k < tr.ntiles && !*abort_flag; ++k) {
        if (tr.ragged_last && k == tr.ntiles - 1) break;    // CUDA-core value sum for a partial page
        const int lp = tr.t_begin / kTile + k;
        const int pg = page_of(a, b, lp);
        const int row0 = pg < 0 ? rows_total : (pg * a.G + g) * a.P;
        for (int mb = 0; mb < NRV; ++mb) {
          for (int th = 0; th < 2; ++th) {
            if (!mbar_wait(bar(BAR_ZV_EMPTY + stage), phase ^ 1, abort_flag, st, 11)) break;
            mbar_expect_tx(bar(BAR_ZV_FULL + stage), kZvBytes);
            const uint32_t dst = base + L.zv + stage * kZvBytes;
            tma_load_2d(dst, &tm_zv, mb * 128, row0 + th * 64, bar(BAR_ZV_FULL + stage));
            tma_load_2d(dst + 8192, &tm_zv, mb * 128 + 64, row0 + th * 64, bar(BAR_ZV_FULL + stage));
            if (++stage == kNVS) { stage = 0; phase ^= 1; }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      constexpr int kBf = ACT == PALU_BF16 ? 1 : 0;
      const uint32_t idesc_d = idesc_f16(kBf, 0, 1, 256, 128);    // z_k K-major, B_k MN-major
      const uint32_t idesc_pv = idesc_f16(kBf, 1, 0, 16, 128);    // z_vᵀ MN-major, Pᵀ K-major
      const uint32_t b_lbo = (uint32_t)a.r_k * 128;                // bytes between 64-column blocks of B
      int zs = 0, vs = 0;
      uint32_t zph = 0, vph = 0;
      bool ok = mbar_wait(bar(BAR_B), 0, abort_flag, st, 20);

      auto issue_pv = [&](int j) -> bool {
        if (!mbar_wait(bar(BAR_P_FULL + (j & 1)), (j >> 1) & 1, abort_flag, st, 21)) return false;
        tc_fence_after();
        const uint32_t a_tmem = tmem + (uint32_t)(j & 1) * 256;
        for (int mb = 0; mb < NRV; ++mb) {
          for (int th = 0; th < 2; ++th) {
            if (!mbar_wait(bar(BAR_ZV_FULL + vs), vph, abort_flag, st, 22)) return false;
            tc_fence_after();
            const uint32_t zv_addr = base + L.zv + vs * kZvBytes;
            const uint32_t p_addr = base + L.p + (uint32_t)(j & 1) * kPBytes + th * 2048;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sdesc_sw128(zv_addr + kk * 16 * 128, 8192, 1024);
              const uint64_t bd = sdesc_sw128(p_addr + kk * 32, 16, 1024);
              umma_f16(a_tmem + mb * 16, ad, bd, idesc_pv, (th | kk) != 0);
            }
            umma_commit(bar(BAR_ZV_EMPTY + vs));
            if (++vs == kNVS) { vs = 0; vph ^= 1; }
          }
        }
        umma_commit(bar(BAR_AT_FULL));
        return true;
      };

      for (int k = 0; k < tr.ntiles && ok; ++k) {
        const int slot = k & 1;
        if (!mbar_wait(bar(BAR_D_EMPTY + slot), ((k >> 1) & 1) ^ 1, abort_flag, st, 23)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)slot * 256;
        const int pv_at = nkc >= 2 ? nkc - 2 : 0;
        for (int c = 0; c < nkc; ++c) {
          if (!mbar_wait(bar(BAR_ZK_FULL + zs), zph, abort_flag, st, 24)) { ok = false; break; }
          tc_fence_after();
          const uint32_t zk_addr = base + L.zk + zs * kZkBytes;
          const uint32_t b_addr = base + L.b + (uint32_t)c * kChunk * 128;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sdesc_sw128(zk_addr + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b_addr + kk * 16 * 128, b_lbo, 1024);
            umma_f16(d_tmem, ad, bd, idesc_d, (c | kk) != 0);
          }
          umma_commit(bar(BAR_ZK_EMPTY + zs));
          if (++zs == kNKS) { zs = 0; zph ^= 1; }
          if (c == pv_at && k >= 1 && !(tr.ragged_last && k - 1 == tr.ntiles - 1)) {
            if (!issue_pv(k - 1)) { ok = false; break; }
          }
        }
        if (!ok) break;
        umma_commit(bar(BAR_D_FULL + slot));
      }
      if (ok && tr.ntiles > 0 && !tr.ragged_last) ok = issue_pv(tr.ntiles - 1);
      // drain: every MMA issued above has completed before TMEM is released
      umma_commit(bar(BAR_TEARDOWN));
      mbar_wait(bar(BAR_TEARDOWN), 0, abort_flag, st, 25);
    }
  } else {
    // ============================================================ epilogue (warps 2-5)
    const int q4 = warp & 3;                 // TMEM lane quarter this warp may access
    const int row = q4 * 32 + lane;          // token row of the tile / latent row of aᵀ
    const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
    float* qr = reinterpret_cast<float*>(sbase + L.qr);
    const uint64_t* om = reinterpret_cast<const uint64_t*>(sbase + L.omega);
    const int head0 = g * a.gs + hp * 2;
    constexpr float kLog2e = 1.4426950408889634f;
    // All 128 epilogue threads meet here; a bounded wait (unlike bar.sync), so a
    // thread that gave up on a timed-out wait cannot strand the others.
    uint32_t epi_phase = 0;
    auto ep_sync = [&](int where) -> bool {
      mbar_arrive(bar(BAR_EPI));
      const bool r = mbar_wait(bar(BAR_EPI), epi_phase, abort_flag, st, where);
      epi_phase ^= 1;
      return r;
    };
    // rotated query of both heads, scaled by log2(e)/sqrt(d_h) for exp2
    {
      const int hh = row >> 6, i = row & 63;
      using TA = typename Dt<ACT>::T;
      const TA* qh = reinterpret_cast<const TA*>(a.q) + ((size_t)b * a.H + head0 + hh) * 128;
      const float x1 = Dt<ACT>::to_f(qh[i]), x2 = Dt<ACT>::to_f(qh[i + 64]);
      float c = 1.f, s = 0.f;
      if (a.rope) rope_cs_fast(a.q_pos[b], a.omega[i], c, s);
      const float sc = a.sm_scale * kLog2e;
      qr[hh * 128 + i] = (x1 * c - x2 * s) * sc;
      qr[hh * 128 + i + 64] = (x2 * c + x1 * s) * sc;
    }
    bool ok = ep_sync(32);

    float m_run[2] = {-INFINITY, -INFINITY};
    float l_part[2] = {0.f, 0.f};
    float acc[2][NRV];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
      for (int mb = 0; mb < NRV; ++mb) acc[hh][mb] = 0.f;
    float prev_scale[2] = {0.f, 0.f};
    float* red = reinterpret_cast<float*>(sbase + L.red);

    auto fold_at = [&](int j, const float* scale) -> bool {
      if (!mbar_wait(bar(BAR_AT_FULL), j & 1, abort_flag, st, 30)) return false;
      tc_fence_after();
#pragma unroll
      for (int mb = 0; mb < NRV; ++mb) {
        float v[2];
        tmem_ld2(tmem + lane_addr + (uint32_t)(j & 1) * 256 + mb * 16, v);
        tmem_wait_ld();
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) acc[hh][mb] = fmaf(acc[hh][mb], scale[hh], v[hh]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_D_EMPTY + (j & 1)));
      return true;
    };

    for (int k = 0; k < tr.ntiles && ok; ++k) {
      const int t0 = tr.t_begin + k * kTile;
      const bool valid = t0 + row < tr.t_end;
      int pos = t0 + row;
      if (a.pos_pool != nullptr) {
        const int pg = page_of(a, b, t0 / kTile);
        pos = pg >= 0 ? a.pos_pool[(size_t)pg * a.P + row] : 0;
      }
      const int slot = k & 1;
      if (!mbar_wait(bar(BAR_D_FULL + slot), (k >> 1) & 1, abort_flag, st, 31)) { ok = false; break; }
      tc_fence_after();
      float sacc[2] = {0.f, 0.f};
#pragma unroll 1
      for (int j = 0; j < 2; ++j) {
        float cs[32], sn[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          if (a.rope) {
            rope_cs_fast(pos, om[j * 32 + u], cs[u], sn[u]);
          } else {
            cs[u] = 1.f;
            sn[u] = 0.f;
          }
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float lo[32], hi[32];
          const uint32_t col = tmem + lane_addr + (uint32_t)slot * 256 + hh * 128 + j * 32;
          tmem_ld32(col, lo);
          tmem_ld32(col + 64, hi);
          tmem_wait_ld();
          const float* qa = qr + hh * 128 + j * 32;
          float s = 0.f;
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            const float k1 = lo[u] * cs[u] - hi[u] * sn[u];
            const float k2 = hi[u] * cs[u] + lo[u] * sn[u];
            s = fmaf(qa[u], k1, s);
            s = fmaf(qa[u + 64], k2, s);
          }
          sacc[hh] += s;
        }
      }
      tc_fence_before();
      // tile max per head across the 128 tokens
      float sc[2], mt[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        sc[hh] = valid ? sacc[hh] : -INFINITY;
        float m = sc[hh];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (lane == 0) red[(k & 1) * 8 + q4 * 2 + hh] = m;
      }
      if (!ep_sync(33)) { ok = false; break; }
      float scale[2], p[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const float* rr = red + (k & 1) * 8;
        mt[hh] = fmaxf(fmaxf(rr[0 * 2 + hh], rr[1 * 2 + hh]), fmaxf(rr[2 * 2 + hh], rr[3 * 2 + hh]));
        const float m_new = fmaxf(m_run[hh], mt[hh]);
        scale[hh] = exp2f(m_run[hh] - m_new);                 // 0 on the first tile
        const uint16_t pb = to_bits<ACT>(valid ? exp2f(sc[hh] - m_new) : 0.f);
        p[hh] = from_bits<ACT>(pb);
        *reinterpret_cast<uint16_t*>(sbase + L.p + slot * kPBytes + p_offset(hh, row)) = pb;
        l_part[hh] = fmaf(l_part[hh], scale[hh], p[hh]);
        m_run[hh] = m_new;
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_P_FULL + slot));
      if (k >= 1) {
        if (!fold_at(k - 1, prev_scale)) { ok = false; break; }
      }
      prev_scale[0] = scale[0];
      prev_scale[1] = scale[1];
    }

    if (ok && tr.ntiles > 0) {
      const int kl = tr.ntiles - 1;
      if (!tr.ragged_last) {
        ok = fold_at(kl, prev_scale);
      } else {
        // partial last page: a += Σ_{valid tokens} p · z_v on CUDA cores,
        // reading only the valid rows (the rest of the page is never touched)
        ok = ep_sync(34);   // every P entry of this tile is written
        const int t0 = tr.t_begin + kl * kTile;
        const int nvalid = tr.t_end - t0;
        const int pg = page_of(a, b, t0 / kTile);
        using TL = typename Dt<ACT>::T;
        float at[2][NRV];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int mb = 0; mb < NRV; ++mb) at[hh][mb] = 0.f;
        if (pg >= 0) {
          const TL* zv = reinterpret_cast<const TL*>(
              reinterpret_cast<const uint8_t*>(a.zv) + ((size_t)(pg * a.G + g) * a.P) * a.v_row);
          const uint8_t* pb = sbase + L.p + (kl & 1) * kPBytes;
          for (int t = 0; t < nvalid; ++t) {
            const float p0 = from_bits<ACT>(*reinterpret_cast<const uint16_t*>(pb + p_offset(0, t)));
            const float p1 = from_bits<ACT>(*reinterpret_cast<const uint16_t*>(pb + p_offset(1, t)));
#pragma unroll
            for (int mb = 0; mb < NRV; ++mb) {
              const float z = Dt<ACT>::to_f(zv[(size_t)t * a.r_v + mb * 128 + row]);
              at[0][mb] = fmaf(p0, z, at[0][mb]);
              at[1][mb] = fmaf(p1, z, at[1][mb]);
            }
          }
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int mb = 0; mb < NRV; ++mb) acc[hh][mb] = fmaf(acc[hh][mb], prev_scale[hh], at[hh][mb]);
      }
    }

    // l: sum of the per-thread partials of each head
    float* lred = reinterpret_cast<float*>(sbase + L.lred);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float v = l_part[hh];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0) lred[q4 * 2 + hh] = v;
    }
    ok = ep_sync(35) && ok;
    if (ok && !*abort_flag) {
      constexpr float kLn2 = 0.6931471805599453f;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float* out = a.part + (((size_t)b * a.H + head0 + hh) * a.S + blockIdx.x) * (a.r_v + 2);
        if (row == 0) {
          out[0] = tr.ntiles > 0 ? m_run[hh] * kLn2 : -INFINITY;
          out[1] = lred[0 * 2 + hh] + lred[1 * 2 + hh] + lred[2 * 2 + hh] + lred[3 * 2 + hh];
        }
#pragma unroll
        for (int mb = 0; mb < NRV; ++mb) out[2 + mb * 128 + row] = acc[hh][mb];
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_map_2d(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, int elt_bytes, uint64_t inner,
                 uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  (void)elt_bytes;
  CUresult r = fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int ACT, int NRV>
cudaError_t launch_t(const DecodeArgs& a, cudaStream_t st) {
  const CUtensorMapDataType dt = ACT == PALU_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const uint64_t rows = (uint64_t)a.num_pages * a.G * a.P;
  CUtensorMap tm_zk, tm_zv, tm_bk;
  if (!make_map_2d(&tm_zk, a.zk, dt, 2, a.r_k, rows, (uint64_t)a.r_k * 2, 64, 128) ||
      !make_map_2d(&tm_zv, a.zv, dt, 2, a.r_v, rows, (uint64_t)a.r_v * 2, 64, 64) ||
      !make_map_2d(&tm_bk, a.Bk, dt, 2, a.W, (uint64_t)a.G * a.r_k, (uint64_t)a.W * 2, 64, a.r_k))
    return cudaErrorInvalidValue;
  const Smem L = smem_layout(a.r_k);
  const size_t smem = L.total + 1024;
  auto kern = decode_tc_kernel<ACT, NRV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.S, a.G * (a.gs / 2), a.batch);
  kern<<<grid, kThreads, smem, st>>>(tm_zk, tm_zv, tm_bk, a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

bool tc_decode_supported(const palu_config* c) {
  if (c->head_dim != 128 || c->page_size != kTile) return false;
  if (c->group_size % 2 != 0) return false;
  if (c->act_dtype != PALU_F16 && c->act_dtype != PALU_BF16) return false;
  if (c->latent_dtype != c->act_dtype) return false;
  if (c->rank_k % kChunk != 0 || c->rank_k > 256) return false;
  if (c->rank_v != 128 && c->rank_v != 256) return false;
  const Smem L = smem_layout(c->rank_k);
  return L.total + 1024 <= 227 * 1024;
}

int tc_head_blocks(const palu_config* c) { return c->group_size / 2; }

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st) {
  if (a.gs % 2 != 0) return cudaErrorInvalidValue;
  if (a.act == PALU_BF16) return a.r_v == 256 ? launch_t<PALU_BF16, 2>(a, st) : launch_t<PALU_BF16, 1>(a, st);
  return a.r_v == 256 ? launch_t<PALU_F16, 2>(a, st) : launch_t<PALU_F16, 1>(a, st);
}

}  // namespace palu
