// Tensor-core compress / append (sm_100a): z = x · A into the paged latent cache.
//
// Method: "PALU 论文低秩投影分解" §低秩投影分解 (z_k = x A_k, z_v = x A_v) and
// §把它放进一次真实推理流程里看, Prefill 阶段 (compute the latents and cache them).
//
// The GEMM runs transposed: D[128 latent columns × NT tokens] = Aᵀ · xᵀ, so the
// TMEM lane of an epilogue thread is one latent column and its TMEM columns are
// tokens.  A thread then writes its column of every token straight into the
// paged, swizzled cache, and for int4 the 32 lanes of a warp are exactly one
// 32-entry quantisation block (max by warp shuffle).
//
// Prefill (many tokens): one CTA per (column tile, 256-token tile), full K.
// Append (a few tokens per decode step): the whole step is one token tile and
// the K range is split across CTAs so the weight matrix streams from every SM;
// each split writes its fp32 partial to the workspace and the last split of a
// column tile (atomic counter) sums them and runs the epilogue.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "palu_common.cuh"
#include "palu_internal.h"
#include "palu_tc.h"
#include "tc_ptx.cuh"

namespace palu {
namespace {

using namespace tc;

constexpr int kThreads = 192;           // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kM = 128;                 // latent columns per tile
constexpr int kKStage = 64;             // K rows per stage
constexpr int kABytes = kM * kKStage * 2;  // 16 KB: two 64-column MN-major boxes

struct Plan {
  int NT;       // tokens per tile (multiple of 16, <= 256)
  int ntt;      // token tiles
  int tk, tv;   // column tiles of A_k and A_v
  int KS;       // K splits
  int stages;
  size_t counter_bytes, partial_bytes;
};

// ncols_k / ncols_v: the launch's output columns on the key and value sides
Plan make_plan(int n, int d_model, int ncols_k, int ncols_v) {
  Plan p{};
  p.NT = n <= 256 ? ((n + 15) / 16) * 16 : 256;
  p.ntt = (n + p.NT - 1) / p.NT;
  p.tk = (ncols_k + kM - 1) / kM;
  p.tv = (ncols_v + kM - 1) / kM;
  const int tiles = (p.tk + p.tv) * p.ntt;
  const int kst = d_model / kKStage;
  int ks = 1;
  if (p.ntt == 1) {
    // an append (one token tile): split K so that every column tile streams A from
    // its own SMs, all CTAs in one round (one CTA per SM)
    ks = 148 / tiles;
    if (ks > kst / 2) ks = kst / 2;   // at least two stages per split
    if (ks > 16) ks = 16;
    if (ks < 1) ks = 1;
  }
  p.KS = ks;
  const int stage_bytes = kABytes + p.NT * 128;
  p.stages = (200 * 1024) / stage_bytes;
  if (p.stages > 8) p.stages = 8;
  if (p.stages < 2) p.stages = 2;
  p.counter_bytes = p.KS > 1 ? ((size_t)tiles * sizeof(int) + 255) / 256 * 256 : 0;
  p.partial_bytes = p.KS > 1 ? (size_t)p.KS * tiles * kM * p.NT * sizeof(float) : 0;
  return p;
}

struct TcArgs {
  CompressArgs a;
  Plan p;
  int* counters;
  float* partials;
};

// Column of A holding output column lc of this launch (entry e = the column
// table's entry of lc, latent entry lc - cols[e]).  Past the last entry it
// continues from the last one, so a TMA box that runs off the end still has a
// valid start (those columns are computed and dropped).  Entries are multiples
// of 64 columns wide, so a 64-column box never straddles two.
__device__ __forceinline__ int a_column(const GroupMap& gm, const uint16_t* cols, const uint16_t* row0, int lc) {
  const int e = col_entry(cols, gm.n, lc);
  return row0[e] + (lc - cols[e]);
}

// Where the tokens of a tile go: page (slot / P, or -1 for a token that is not
// stored) and row (slot % P) of every token, filled once per tile into shared
// memory by the epilogue threads, so the per-token stores never wait on a
// dependent load of the slot mapping.  An out-of-range slot is reported.
__device__ __forceinline__ void fill_token_table(const CompressArgs& a, int t0, int ntok, int2* tab, int tid,
                                                 int nthr, DevStatus* st) {
  const long long cap = (long long)a.num_pages * a.P;
  for (int i = tid; i < ntok; i += nthr) {
    const int slot = a.slots[t0 + i];
    int2 d = make_int2(-1, 0);
    if (slot >= cap) report(st, PALU_ERR_DEVICE_BOUNDS, 3000000 + t0 + i);
    else if (slot >= 0) d = make_int2(slot / a.P, slot % a.P);
    tab[i] = d;
  }
}

// The fixed part of this thread's latent column in the paged cache: its group's
// pool, the column block and 16-byte unit of its entry (before the token's
// swizzle), and for int4 the scale pool.  Latent entry j of token row t sits at
// block (j·es / 128)·P·128 + t·128 + (((j·es / 16) mod 8) xor (t mod 8))·16 + j·es mod 16.
struct ColDst {
  uint8_t* col;          // pool + page-independent part of the offset
  long long page_bytes;  // stride between pages
  int unit;              // 16-byte unit before the swizzle
  bool ok;               // a real column of this launch
  uint8_t* spool;        // int4: scale pool + this column's scale slot
  long long spage, srow;
};

template <int LAT>
__device__ __forceinline__ ColDst col_dst(const CompressArgs& a, bool is_v, const uint16_t* cols, int ncols, int gc) {
  ColDst d{};
  d.ok = gc < ncols;
  const int e = d.ok ? col_entry(cols, a.gm.n, gc) : 0;   // group entry of this column
  const int j = d.ok ? gc - cols[e] : 0;                    // latent entry within it
  long long o = j >> 1;                                     // int4: two entries per byte
  if constexpr (LAT != PALU_INT4) o = (long long)j * (long long)sizeof(typename Dt<LAT>::T);
  d.col = const_cast<uint8_t*>(is_v ? a.gm.zv[e] : a.gm.zk[e]) + (o >> 7) * (long long)a.P * 128 + (o & 15);
  d.page_bytes = is_v ? a.gm.v_page : a.gm.k_page;
  d.unit = (int)((o >> 4) & 7);
  if constexpr (LAT == PALU_INT4) {
    d.spool = const_cast<uint8_t*>(is_v ? a.gm.zvs[e] : a.gm.zks[e]) + 2 * (j >> 5);
    d.spage = is_v ? a.gm.vs_page : a.gm.ks_page;
    d.srow = int4_scale_row(cols[e + 1] - cols[e]);
  }
  return d;
}

// Write 16 tokens (tile rows j0 .. j0 + 15, fewer at the end) of this thread's
// latent column (its warp holds 32 consecutive columns) into the paged cache:
// rounded to the latent dtype, or int4-quantised per 32-column block.
template <int LAT>
__device__ __forceinline__ void store_tokens(const ColDst& cd, const int2* tab, int j0, int ntok, const float* v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    if (j0 + u >= ntok) break;
    const int2 d = tab[j0 + u];   // the same entry in every lane: warp-uniform branches
    if (d.x < 0) continue;
    uint8_t* dst = cd.col + (long long)d.x * cd.page_bytes + d.y * 128 + ((cd.unit ^ (d.y & 7)) << 4);
    if constexpr (LAT == PALU_INT4) {
      // the warp's 32 columns are one quantisation block of this token
      float amax = cd.ok ? fabsf(v[u]) : 0.f;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const __half s16 = __float2half_rn(__fdiv_rn(amax, 7.0f));
      const float s = __half2float(s16);
      int code = 0;
      if (s != 0.f) code = (int)fminf(fmaxf(rintf(__fdiv_rn(v[u], s)), -7.f), 7.f);
      const int hi = __shfl_down_sync(0xffffffffu, code, 1);
      if (cd.ok && (lane & 1) == 0) *dst = (uint8_t)((code & 0xF) | ((hi & 0xF) << 4));
      if (cd.ok && lane == 0)
        *reinterpret_cast<__half*>(cd.spool + (long long)d.x * cd.spage + d.y * cd.srow) = s16;
    } else {
      if (cd.ok) *reinterpret_cast<typename Dt<LAT>::T*>(dst) = Dt<LAT>::from_f(v[u]);
    }
  }
}

template <int ACT, int LAT>
__global__ void __launch_bounds__(kThreads, 1)
    compress_tc_kernel(const __grid_constant__ CUtensorMap tm_ak, const __grid_constant__ CUtensorMap tm_av,
                       const __grid_constant__ CUtensorMap tm_x, const TcArgs t) {
  extern __shared__ uint8_t smem_raw[];
  const CompressArgs& a = t.a;
  const Plan& p = t.p;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  const int stage_bytes = kABytes + p.NT * 128;
  const uint32_t bars = base + (uint32_t)p.stages * stage_bytes;      // 2·stages + 2 barriers
  uint8_t* misc = sbase + (uint32_t)p.stages * stage_bytes + 256;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 16);
  int* last_flag = reinterpret_cast<int*>(misc + 32);
  int2* tok_tab = reinterpret_cast<int2*>(misc + 64);   // NT entries
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (p.stages + s); };
  const uint32_t d_full = bars + 8u * (2 * p.stages);
  const uint32_t epi_bar = d_full + 8;
  const uint32_t td_bar = d_full + 16;   // teardown: every MMA of the CTA has completed
  DevStatus* st = reinterpret_cast<DevStatus*>(a.status);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // tile coordinates
  const bool is_v = blockIdx.x >= p.tk;
  const int ctile = is_v ? blockIdx.x - p.tk : blockIdx.x;
  const int c0 = ctile * kM;
  const uint16_t* cols = is_v ? a.vcol : a.kcol;
  const int ncols = is_v ? a.ncols_v : a.ncols_k;
  const int t0 = blockIdx.y * p.NT;
  const int kst = a.d_model / kKStage;
  const int split = blockIdx.z;
  const int ks0 = (int)((long long)kst * split / p.KS), ks1 = (int)((long long)kst * (split + 1) / p.KS);
  const CUtensorMap* tm_a = is_v ? &tm_av : &tm_ak;

  if (threadIdx.x == 0) {
    abort_init(abort_flag, a.wait_cycles);
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    mbar_init(d_full, 1);
    mbar_init(epi_bar, 4);
    mbar_init(td_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(tm_a);
      prefetch_tmap(&tm_x);
      int s = 0;
      uint32_t ph = 0;
      // the tile's two 64-column boxes of A, fixed over the K loop
      const uint16_t* row0 = is_v ? a.gm.v_row0 : a.gm.k_row0;
      const int ax0 = a_column(a.gm, cols, row0, c0), ax1 = a_column(a.gm, cols, row0, c0 + 64);
      long long issued = 0;
      for (int kb = ks0; kb < ks1 && !*abort_flag; ++kb) {
        if (!mbar_wait(empty(s), ph ^ 1, abort_flag, st, 50)) break;
        mbar_expect_tx(full(s), (uint32_t)stage_bytes);
        const uint32_t dst = base + (uint32_t)s * stage_bytes;
        tma_load_2d(dst, tm_a, ax0, kb * kKStage, full(s));
        tma_load_2d(dst + kABytes / 2, tm_a, ax1, kb * kKStage, full(s));
        tma_load_2d(dst + kABytes, &tm_x, kb * kKStage, t0, full(s));
        ++issued;
        if (++s == p.stages) { s = 0; ph ^= 1; }
      }
      // after an abort, loads already issued still land in shared memory: wait for them
      drain_ring(full(0), p.stages, issued, st, 50);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr int kBf = ACT == PALU_BF16 ? 1 : 0;
      const uint32_t idesc = idesc_f16(kBf, 1, 0, p.NT, kM);    // Aᵀ MN-major, xᵀ K-major
      int s = 0;
      uint32_t ph = 0;
      // timeout-path test hook: first wait on a phase nothing completes before the teardown commit
      bool ok = a.stall_test == 0 || mbar_wait(td_bar, 0, abort_flag, st, 55);
      for (int kb = ks0; kb < ks1 && ok; ++kb) {
        if (!mbar_wait(full(s), ph, abort_flag, st, 51)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = base + (uint32_t)s * stage_bytes;
        const uint32_t sx = sa + kABytes;
#pragma unroll
        for (int kk = 0; kk < kKStage / 16; ++kk) {
          const uint64_t ad = sdesc(sa + kk * 16 * 128, kABytes / 2, 1024, kSw128);
          const uint64_t bd = sdesc(sx + kk * 32, 16, 1024, kSw128);
          umma_f16(tmem, ad, bd, idesc, (kb > ks0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(empty(s));
        if (++s == p.stages) { s = 0; ph ^= 1; }
      }
      if (ok) umma_commit(d_full);   // fires once every MMA above has completed
      // drain, also after an abort: every MMA issued completes before TMEM is released
      umma_commit(td_bar);
      mbar_drain(td_bar, 0, st, 56);
    }
  } else {
    // ============================================================ epilogue (warps 2-5)
    const int q4 = warp & 3;
    const int c = q4 * 32 + lane;            // latent column of this thread within the tile
    const int gc = c0 + c;
    const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
    uint32_t epi_phase = 0;
    auto ep_sync = [&](int where) -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_bar);
      const bool rr = mbar_wait(epi_bar, epi_phase, abort_flag, st, where);
      epi_phase ^= 1;
      return rr;
    };
    // the tokens' destinations, while the MMAs run; published by the syncs below
    const int ntok = min(p.NT, a.n - t0);
    fill_token_table(a, t0, ntok, tok_tab, threadIdx.x - 64, kThreads - 64, st);
    bool ok = mbar_wait(d_full, 0, abort_flag, st, 52);
    tc_fence_after();
    const int tile_id = blockIdx.x * p.ntt + blockIdx.y;
    const int tiles = (p.tk + p.tv) * p.ntt;
    bool finalize = true;
    float* my_part = nullptr;
    if (p.KS > 1) {
      // publish this split's partial, then find out whether this CTA closes the tile
      my_part = t.partials + ((size_t)split * tiles + tile_id) * kM * p.NT + (size_t)c * p.NT;
      for (int j0 = 0; ok && j0 < p.NT; j0 += 16) {
        float v[16];
        tmem_ld16(tmem + lane_addr + j0, v);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; u += 4)
          *reinterpret_cast<float4*>(my_part + j0 + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
      }
      __threadfence();
      ok = ep_sync(53) && ok;
      if (threadIdx.x == 64) {
        // a CTA that gave up neither counts itself nor closes the tile
        const int prev = ok ? atomicAdd(t.counters + tile_id, 1) : -1;
        *last_flag = (prev == p.KS - 1);
      }
      ok = ep_sync(54) && ok;
      finalize = *last_flag != 0;
      if (finalize) __threadfence();
    }
    if (p.KS == 1) ok = ep_sync(57) && ok;
    if (ok && finalize) {
      const ColDst cd = col_dst<LAT>(a, is_v, cols, ncols, gc);
      for (int j0 = 0; j0 < ntok; j0 += 16) {
        float v[16];
        if (p.KS == 1) {
          tmem_ld16(tmem + lane_addr + j0, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int u = 0; u < 16; ++u) v[u] = 0.f;
          for (int sp = 0; sp < p.KS; ++sp) {
            const float* src = t.partials + ((size_t)sp * tiles + tile_id) * kM * p.NT + (size_t)c * p.NT + j0;
#pragma unroll
            for (int u = 0; u < 16; u += 4) {
              const float4 f = __ldcg(reinterpret_cast<const float4*>(src + u));
              v[u] += f.x;
              v[u + 1] += f.y;
              v[u + 2] += f.z;
              v[u + 3] += f.w;
            }
          }
        }
        store_tokens<LAT>(cd, tok_tab, j0, ntok, v);
      }
      // positions, once per token
      if (!is_v && ctile == 0 && a.positions != nullptr && a.pos_pool != nullptr) {
        for (int i = c; i < ntok; i += kM) {
          const int2 d = tok_tab[i];
          if (d.x >= 0) a.pos_pool[(long long)d.x * a.P + d.y] = a.positions[t0 + i];
        }
      }
      if (p.KS > 1 && threadIdx.x == 64) t.counters[tile_id] = 0;   // reusable for the next call
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// Prefill (several token tiles, no K split): a persistent kernel, one CTA per SM,
// walking the (column tile, token tile) tiles round-robin with two TMEM
// accumulators, so that the epilogue of one tile overlaps the MMAs of the next.
// Consecutive tiles share their token tile (x stays in L2 while the column tiles
// pass over it).  Same roles as above: warp 0 TMA, warp 1 MMA, warps 2-5 epilogue.
template <int ACT, int LAT>
__global__ void __launch_bounds__(kThreads, 1)
    compress_tc_persistent_kernel(const __grid_constant__ CUtensorMap tm_ak, const __grid_constant__ CUtensorMap tm_av,
                                  const __grid_constant__ CUtensorMap tm_x, const TcArgs t) {
  extern __shared__ uint8_t smem_raw[];
  const CompressArgs& a = t.a;
  const Plan& p = t.p;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  const int stage_bytes = kABytes + p.NT * 128;
  const uint32_t bars = base + (uint32_t)p.stages * stage_bytes;      // 2·stages + 6 barriers
  uint8_t* misc = sbase + (uint32_t)p.stages * stage_bytes + 256;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 16);
  int2* tok_tab = reinterpret_cast<int2*>(misc + 64);   // 2 × NT entries, by tile parity
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (p.stages + s); };
  auto acc_full = [&](int b) { return bars + 8u * (2 * p.stages + b); };
  auto acc_empty = [&](int b) { return bars + 8u * (2 * p.stages + 2 + b); };
  const uint32_t td_bar = bars + 8u * (2 * p.stages + 4);   // teardown: every MMA has completed
  const uint32_t epi_bar = bars + 8u * (2 * p.stages + 5);  // the 4 epilogue warps: token table written
  DevStatus* st = reinterpret_cast<DevStatus*>(a.status);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ctiles = p.tk + p.tv;
  const int ntiles = ctiles * p.ntt;
  const int kst = a.d_model / kKStage;
  // tile i of this CTA: global tile blockIdx.x + i·gridDim.x = (column tile, token tile)
  auto tile_of = [&](int i, int& ctile, bool& is_v, int& c0, int& t0) {
    const int tg = blockIdx.x + i * gridDim.x;
    const int ct = tg % ctiles;
    is_v = ct >= p.tk;
    ctile = is_v ? ct - p.tk : ct;
    c0 = ctile * kM;
    t0 = (tg / ctiles) * p.NT;
  };
  const int my_tiles = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (threadIdx.x == 0) {
    abort_init(abort_flag, a.wait_cycles);
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full(b), 1);
      mbar_init(acc_empty(b), 4);
    }
    mbar_init(td_bar, 1);
    mbar_init(epi_bar, 4);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_ak);
      prefetch_tmap(&tm_av);
      prefetch_tmap(&tm_x);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      long long issued = 0;
      for (int i = 0; i < my_tiles && ok; ++i) {
        int ctile, c0, t0;
        bool is_v;
        tile_of(i, ctile, is_v, c0, t0);
        const CUtensorMap* tm_a = is_v ? &tm_av : &tm_ak;
        const uint16_t* cols = is_v ? a.vcol : a.kcol;
        const uint16_t* row0 = is_v ? a.gm.v_row0 : a.gm.k_row0;
        const int ax0 = a_column(a.gm, cols, row0, c0), ax1 = a_column(a.gm, cols, row0, c0 + 64);
        for (int kb = 0; kb < kst; ++kb) {
          if (*abort_flag || !mbar_wait(empty(s), ph ^ 1, abort_flag, st, 60)) { ok = false; break; }
          mbar_expect_tx(full(s), (uint32_t)stage_bytes);
          const uint32_t dst = base + (uint32_t)s * stage_bytes;
          tma_load_2d(dst, tm_a, ax0, kb * kKStage, full(s));
          tma_load_2d(dst + kABytes / 2, tm_a, ax1, kb * kKStage, full(s));
          tma_load_2d(dst + kABytes, &tm_x, kb * kKStage, t0, full(s));
          ++issued;
          if (++s == p.stages) { s = 0; ph ^= 1; }
        }
      }
      // after an abort, loads already issued still land in shared memory: wait for them
      drain_ring(full(0), p.stages, issued, st, 60);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr int kBf = ACT == PALU_BF16 ? 1 : 0;
      const uint32_t idesc = idesc_f16(kBf, 1, 0, p.NT, kM);    // Aᵀ MN-major, xᵀ K-major
      int s = 0;
      uint32_t ph = 0;
      // timeout-path test hook: first wait on a phase nothing completes before the teardown commit
      bool ok = a.stall_test == 0 || mbar_wait(td_bar, 0, abort_flag, st, 65);
      for (int i = 0; i < my_tiles && ok; ++i) {
        const int b = i & 1;
        // the epilogue has read this accumulator's previous tile (i - 2)
        if (!mbar_wait(acc_empty(b), ((i >> 1) & 1) ^ 1, abort_flag, st, 61)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + 256u * b;
        for (int kb = 0; kb < kst; ++kb) {
          if (!mbar_wait(full(s), ph, abort_flag, st, 62)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = base + (uint32_t)s * stage_bytes;
          const uint32_t sx = sa + kABytes;
#pragma unroll
          for (int kk = 0; kk < kKStage / 16; ++kk) {
            const uint64_t ad = sdesc(sa + kk * 16 * 128, kABytes / 2, 1024, kSw128);
            const uint64_t bd = sdesc(sx + kk * 32, 16, 1024, kSw128);
            umma_f16(d, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(empty(s));
          if (++s == p.stages) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        umma_commit(acc_full(b));   // fires once every MMA of the tile has completed
      }
      // drain, also after an abort: every MMA issued completes before TMEM is released
      umma_commit(td_bar);
      mbar_drain(td_bar, 0, st, 63);
    }
  } else {
    // ============================================================ epilogue (warps 2-5)
    const int q4 = warp & 3;
    const int c = q4 * 32 + lane;            // latent column of this thread within the tile
    const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
    for (int i = 0; i < my_tiles; ++i) {
      const int b = i & 1;
      int ctile, c0, t0;
      bool is_v;
      tile_of(i, ctile, is_v, c0, t0);
      const int ntok = min(p.NT, a.n - t0);
      // the token table of tile i (its parity's half; the other half may still be read
      // for tile i - 1 by a slower warp, which has passed this sync only after it)
      int2* tab = tok_tab + b * p.NT;
      fill_token_table(a, t0, ntok, tab, threadIdx.x - 64, kThreads - 64, st);
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_bar);
      if (!mbar_wait(epi_bar, (uint32_t)(i & 1), abort_flag, st, 66)) break;
      const uint16_t* cols = is_v ? a.vcol : a.kcol;
      const int ncols = is_v ? a.ncols_v : a.ncols_k;
      const ColDst cd = col_dst<LAT>(a, is_v, cols, ncols, c0 + c);
      if (!mbar_wait(acc_full(b), (i >> 1) & 1, abort_flag, st, 64)) break;
      tc_fence_after();
      for (int j0 = 0; j0 < ntok; j0 += 16) {
        float v[16];
        tmem_ld16(tmem + lane_addr + 256u * b + j0, v);
        tmem_wait_ld();
        store_tokens<LAT>(cd, tab, j0, ntok, v);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty(b));
      // positions, once per token
      if (!is_v && ctile == 0 && a.positions != nullptr && a.pos_pool != nullptr) {
        for (int k = c; k < ntok; k += kM) {
          const int2 d = tab[k];
          if (d.x >= 0) a.pos_pool[(long long)d.x * a.P + d.y] = a.positions[t0 + k];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool map2d(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
           uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int ACT, int LAT>
cudaError_t launch_t(const CompressArgs& a, cudaStream_t st) {
  const Plan p = make_plan(a.n, a.d_model, a.ncols_k, a.ncols_v);
  const CUtensorMapDataType dt = ACT == PALU_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap tm_ak, tm_av, tm_x;
  if (!map2d(&tm_ak, a.Ak, dt, (uint64_t)a.a_kcols, a.d_model, (uint64_t)a.a_kcols * 2, 64, kKStage) ||
      !map2d(&tm_av, a.Av, dt, (uint64_t)a.a_vcols, a.d_model, (uint64_t)a.a_vcols * 2, 64, kKStage) ||
      !map2d(&tm_x, a.x, dt, a.d_model, a.n, (uint64_t)a.d_model * 2, 64, p.NT))
    return cudaErrorInvalidValue;
  TcArgs t{};
  t.a = a;
  t.p = p;
  uint8_t* scratch = reinterpret_cast<uint8_t*>(a.scratch);
  t.counters = reinterpret_cast<int*>(scratch);
  t.partials = reinterpret_cast<float*>(scratch + p.counter_bytes);
  // stages, barriers (256), flags (64), token tables (2 × NT), alignment
  const size_t smem = (size_t)p.stages * (kABytes + p.NT * 128) + 256 + 64 + 2 * (size_t)p.NT * sizeof(int2) + 1024;
  if (p.ntt >= 2 && p.KS == 1) {
    // prefill: persistent, one CTA per SM over every tile
    auto kern = compress_tc_persistent_kernel<ACT, LAT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int tiles = (p.tk + p.tv) * p.ntt;
    kern<<<tiles < 148 ? tiles : 148, kThreads, smem, st>>>(tm_ak, tm_av, tm_x, t);
    count_launch();
    return cudaGetLastError();
  }
  auto kern = compress_tc_kernel<ACT, LAT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.tk + p.tv, p.ntt, p.KS);
  kern<<<grid, kThreads, smem, st>>>(tm_ak, tm_av, tm_x, t);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

bool tc_compress_supported(const palu_config* c, int n_tokens, int d_model) {
  if (c->act_dtype != PALU_F16 && c->act_dtype != PALU_BF16) return false;
  if (c->latent_dtype != c->act_dtype && c->latent_dtype != PALU_INT4) return false;
  if (d_model % kKStage != 0 || d_model < 2 * kKStage) return false;
  if (n_tokens <= 0) return false;
  const int G = c->num_heads / c->group_size;
  if ((G * c->rank_k) % 8 != 0 || (G * c->rank_v) % 8 != 0) return false;
  if (c->latent_dtype == PALU_INT4 && (c->rank_k % 32 != 0 || c->rank_v % 32 != 0)) return false;
  return true;
}

size_t tc_compress_scratch_bytes(const palu_config* c, int n_tokens, int d_model, int ncols_k, int ncols_v) {
  if (!tc_compress_supported(c, n_tokens, d_model)) return 0;
  const Plan p = make_plan(n_tokens, d_model, ncols_k, ncols_v);
  return p.counter_bytes + p.partial_bytes;
}

cudaError_t launch_compress_tc(const CompressArgs& a, cudaStream_t st) {
  if (a.act == PALU_BF16) {
    if (a.lat == PALU_INT4) return launch_t<PALU_BF16, PALU_INT4>(a, st);
    return launch_t<PALU_BF16, PALU_BF16>(a, st);
  }
  if (a.lat == PALU_INT4) return launch_t<PALU_F16, PALU_INT4>(a, st);
  return launch_t<PALU_F16, PALU_F16>(a, st);
}

}  // namespace palu
