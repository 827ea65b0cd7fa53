// Fused decode for attention without rotary embedding (sm_100a: tcgen05 + TMEM).
//
// Method: "PALU 论文低秩投影分解" §低秩投影分解 (the latent is either restored
// to full K/V or fused with the operators that follow) and §把它放进一次真实推理
// 流程里看, Decode 阶段 (attention fused with the up-projection, so full K/V are
// never materialised); the v1 abstract of "Palu: Compressing KV-Cache with
// Low-Rank Projection" names matrix fusion.  Without RoPE the key up-projection
// folds into the query:
//   s_{t,h} = q_h · (B_k,hᵀ z_k,t) = (B_k,h q_h) · z_k,t,   B_k,h = B_k[g][:, cols_h],
// so scores come straight from the cached latents and no key is rebuilt; the
// values stay in latent space as on the RoPE path (a = Σ p z_v, then a·B_v in
// the combine).  With RoPE the rotation sits between B_k and q and the fold is
// not available, which is why the main kernel rebuilds keys.
//
// fold_query_kernel: q̃_h = B_k,h q_h · log2(e)/√d_h for the g heads of a group,
//   stored as the sum of two 16-bit numbers (hi + lo) so the tensor cores see
//   q̃ to ~16 significant bits.
// decode_fused_kernel: one CTA per (sequence, group, split), 128 tokens (a page)
//   per tile:
//   warp 0  bulk copies of the z_k and z_v pages through two rings (q̃ is
//           staged into shared memory by all threads at the start);
//   warp 1  MMAs: D[128 tok × 16] = z_k · [q̃_hi ; q̃_lo]ᵀ (scores of the g
//           heads twice, hi and lo parts) and aᵀ[r_v × 16] = z_vᵀ · Pᵀ;
//   warps 2-5  one thread per token / latent row: scores, online softmax of the
//           g heads, P (bf16/fp16), and the fold of aᵀ into running sums.
// Output: per (b, head, split) the partial (m, l, a[r_v]) the combine merges.
#include <cuda.h>
#include <math.h>

#include "palu_common.cuh"
#include "palu_internal.h"
#include "palu_tc.h"
#include "tc_ptx.cuh"

namespace palu {
namespace {

using namespace tc;

constexpr int kTile = 128;          // tokens per tile = page size
constexpr int kChunk = 64;          // K chunk (latent entries) = one 128-byte column block
constexpr int kThreads = 192;       // producer, MMA, four epilogue warps
constexpr int kMaxG = 4;            // heads per group the fused kernel takes
constexpr int kNZK = 6;             // z_k ring stages
constexpr int kNZV = 4;             // z_v ring stages (pairs of column blocks)
constexpr int kStageBytes = kTile * kChunk * 2;   // 16 KB: one column block of a page
constexpr int kFusedMaxQueries = 4;  // queries of one sequence that share a pass over the cache

struct Smem {
  uint32_t qt, zk, zv, p, red, lred, bars, tmem_slot, abort, total;
};

enum {
  BAR_ZK_FULL = 0,
  BAR_ZK_EMPTY = BAR_ZK_FULL + kNZK,
  BAR_ZV_FULL = BAR_ZK_EMPTY + kNZK,
  BAR_ZV_EMPTY = BAR_ZV_FULL + kNZV,
  BAR_D_FULL = BAR_ZV_EMPTY + kNZV,    // 2
  BAR_D_EMPTY = BAR_D_FULL + 2,        // 2
  BAR_P_FULL = BAR_D_EMPTY + 2,        // 2
  BAR_AT_FULL = BAR_P_FULL + 2,        // 2
  BAR_AT_EMPTY = BAR_AT_FULL + 2,      // 2
  BAR_EPI = BAR_AT_EMPTY + 2,          // epilogue warps meet (bounded)
  BAR_TEARDOWN = BAR_EPI + 1,
  BAR_COUNT
};
static_assert(BAR_COUNT <= 32, "barrier space");

__device__ __forceinline__ int page_of(const DecodeArgs& a, int b, int lp) {
  const int pg = a.page_table[(size_t)b * a.max_pages + lp];
  return (pg < 0 || pg >= a.num_pages) ? -1 : pg;
}

template <int ACT>
__device__ __forceinline__ uint16_t to_bits(float v) {
  const auto h = Dt<ACT>::from_f(v);
  return *reinterpret_cast<const uint16_t*>(&h);
}
template <int ACT>
__device__ __forceinline__ float from_bits(uint16_t u) {
  return Dt<ACT>::to_f(*reinterpret_cast<const typename Dt<ACT>::T*>(&u));
}

// q̃ = B_k,h q_h (scaled) for the heads of one group, as hi + lo 16-bit rows:
// out[vb][g][h] = hi, out[vb][g][4 + h] = lo (h < gs; other rows zero), each
// r_k long, for virtual sequence vb = b·qslots + jj (query jj of the pass; a
// single query per step is qslots = 1).  CTA (g, 64 latent entries, 4 virtual
// sequences); thread (entry j, head h) holds the B_k row segment
// B_k[g][j][h·d_h, +d_h) in registers and takes its dot product with each
// query.
constexpr int kFoldSeqs = 4;
template <int ACT>
__global__ void __launch_bounds__(256) fold_query_kernel(const __grid_constant__ DecodeArgs a, int qslots, void* qt) {
  using TA = typename Dt<ACT>::T;
  // rows padded by 4 floats: the four heads' 16-byte reads of one warp land in distinct banks
  __shared__ __align__(16) float qs[kFoldSeqs][kMaxG][128 + 4];
  // blockIdx.x: entry gi of the group map (model group g)
  const int gi = blockIdx.x, jb = blockIdx.y, v0 = blockIdx.z * kFoldSeqs;
  const int g = a.gm.g[gi];
  const int r_k = a.gm.rk[gi];          // this entry's key rank; rows are a.r_k apart
  const int gs = a.gs, d_h = a.d_h;
  const int nvb = a.batch * qslots;
  auto live = [&](int vb) { return vb < nvb && vb % qslots < a.qn; };
  for (int i = threadIdx.x; i < kFoldSeqs * kMaxG * 128; i += blockDim.x) {
    const int bb = i / (kMaxG * 128), h = (i / 128) % kMaxG, d = i % 128;
    const int vb = v0 + bb;
    float v = 0.f;
    if (live(vb) && h < gs && d < d_h)
      v = Dt<ACT>::to_f(reinterpret_cast<const TA*>(a.q)[(size_t)(vb / qslots) * a.q_bstride +
                                                          (size_t)(vb % qslots) * a.H * d_h +
                                                          (size_t)(g * gs + h) * d_h + d]);
    qs[bb][h][d] = v;
  }
  __syncthreads();
  const int jl = threadIdx.x >> 2, h = threadIdx.x & 3;
  const int j = jb * 64 + jl;
  if (j >= r_k) return;
  // the row segment as 8-element vectors (d_h is a multiple of 8 here)
  uint4 bseg[16];
  const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const TA*>(a.Bk) +
                                                    ((size_t)a.gm.k_row0[gi] + j) * a.W + (size_t)h * d_h);
#pragma unroll
  for (int v = 0; v < 16; ++v) bseg[v] = (h < gs && v * 8 < d_h) ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
  constexpr float kLog2e = 1.4426950408889634f;
  const float sc = a.sm_scale * kLog2e;
  for (int bb = 0; bb < kFoldSeqs; ++bb) {
    if (!live(v0 + bb)) continue;
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int v = 0; v < 16; ++v) {
      const TA* e = reinterpret_cast<const TA*>(&bseg[v]);
      const float4 qa = *reinterpret_cast<const float4*>(&qs[bb][h][v * 8]);
      const float4 qb = *reinterpret_cast<const float4*>(&qs[bb][h][v * 8 + 4]);
      acc0 = fmaf(Dt<ACT>::to_f(e[0]), qa.x, acc0);
      acc1 = fmaf(Dt<ACT>::to_f(e[1]), qa.y, acc1);
      acc0 = fmaf(Dt<ACT>::to_f(e[2]), qa.z, acc0);
      acc1 = fmaf(Dt<ACT>::to_f(e[3]), qa.w, acc1);
      acc0 = fmaf(Dt<ACT>::to_f(e[4]), qb.x, acc0);
      acc1 = fmaf(Dt<ACT>::to_f(e[5]), qb.y, acc1);
      acc0 = fmaf(Dt<ACT>::to_f(e[6]), qb.z, acc0);
      acc1 = fmaf(Dt<ACT>::to_f(e[7]), qb.w, acc1);
    }
    float acc = (acc0 + acc1) * sc;
    const TA hi = Dt<ACT>::from_f(acc);
    const TA lo = Dt<ACT>::from_f(acc - Dt<ACT>::to_f(hi));
    TA* out = reinterpret_cast<TA*>(qt) + ((size_t)(v0 + bb) * a.gm.n + gi) * 2 * kMaxG * a.r_k;
    out[(size_t)h * a.r_k + j] = hi;
    out[(size_t)(kMaxG + h) * a.r_k + j] = lo;
  }
}

// Shape of one pass: QN queries of a sequence share each streamed tile.
//   score MMA:  N = 8·QN rows of q̃ (query jj, hi/lo part, head h -> row 8jj + 4·lo + h)
//   value MMA:  N = 4·QN rows of P (query jj, head h -> row 4jj + h), padded to 16
template <int QN>
struct Pass {
  static constexpr int kN = 8 * QN < 16 ? 16 : 8 * QN;
  static constexpr int kPC = kMaxG * QN;                 // (query, head) pairs
  static constexpr int kNP = (kPC + 15) / 16 * 16;
  static constexpr int kPBytes = kNP * kTile * 2;         // P tile: kNP rows × 128 tokens
  static constexpr int kPRegion = kNP * 128;              // bytes per 64 tokens of P
  static constexpr int kAt = 2 * kN;                      // first aᵀ column
  static constexpr int kTmem = 2 * kN + 2 * 2 * kNP <= 128 ? 128 : 256;
};

template <int QN>
__host__ __device__ inline Smem smem_layout(int r_k) {
  using PS = Pass<QN>;
  Smem s{};
  uint32_t o = 0;
  // fixed offsets first; the folded queries (their size follows the key rank) last
  s.zk = o;   o += kNZK * kStageBytes;
  s.zv = o;   o += kNZV * kStageBytes;
  s.p = o;    o += 2 * PS::kPBytes;
  s.red = o;  o += 2 * 4 * PS::kPC * 4;                  // [tile parity][warp][pair] maxima
  s.lred = o; o += 4 * PS::kPC * 4;                      // [warp][pair] softmax denominators
  s.bars = o; o += 32 * 8;
  s.tmem_slot = o; o += 16;
  s.abort = o;     o += 16;
  o = (o + 1023u) & ~1023u;                             // 128-byte-swizzle atoms: 1024-byte aligned
  s.qt = o;   o += (uint32_t)(r_k / kChunk) * PS::kN * 128;   // [K chunk][kN rows][128 B], 128-byte swizzle
  s.total = o;
  return s;
}

// P tile, K-major with the 128-byte swizzle: row n ((query, head) pair), token
// k; tokens 0-63 and 64-127 sit in two atoms of kNP rows.
template <int QN>
__device__ __forceinline__ uint32_t p_offset(int n, int k) {
  const int region = k >> 6, kin = k & 63;
  return (uint32_t)(region * Pass<QN>::kPRegion + n * 128 + (((kin >> 3) ^ (n & 7)) << 4) + (kin & 7) * 2);
}

template <int ACT, int NRV, int QN>
__global__ void __launch_bounds__(kThreads, 1)
    decode_fused_kernel(const __grid_constant__ DecodeArgs a, const void* qt) {
  using PS = Pass<QN>;
  constexpr int kN = PS::kN, kNP = PS::kNP, kPC = PS::kPC, kPB = PS::kPBytes;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  // blockIdx.y: entry gi of the group map (model group gm.g[gi]); its key rank sets the layout
  const int s = blockIdx.x, gi = blockIdx.y, b = blockIdx.z;
  const GroupMap& gm = a.gm;
  const int r_k = gm.rk[gi];
  const Smem L = smem_layout<QN>(r_k);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  DevStatus* st = reinterpret_cast<DevStatus*>(a.status);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + L.abort);
  auto bar = [&](int i) { return base + L.bars + 8u * i; };

  const int gs = a.gs;
  const int nq = a.qn;                  // queries of this pass (<= QN)
  const int nkc = r_k / kChunk;
  int T = a.seq_lens[b];
  const int cap = a.max_pages * a.P;
  if (T < 0 || T > cap) {
    if (threadIdx.x == 0) report(st, PALU_ERR_DEVICE_BOUNDS, 1000000 + b);
    T = T < 0 ? 0 : cap;
  }
  const int npg = (T + kTile - 1) / kTile;
  const int pps = (npg + a.S - 1) / a.S;
  const int pg0 = s * pps;
  const int pg1 = min(npg, pg0 + pps);
  const int ntiles = max(0, pg1 - pg0);
  const int t_end = min(T, pg1 * kTile);
  const bool ragged_last = ntiles > 0 && t_end - (pg0 + ntiles - 1) * kTile < kTile;
  const int nvt = ntiles - (ragged_last ? 1 : 0);   // tiles whose value sum runs on the tensor cores

  if (threadIdx.x == 0) {
    abort_init(abort_flag, a.wait_cycles);
    for (int i = 0; i < kNZK; ++i) {
      mbar_init(bar(BAR_ZK_FULL + i), 1);
      mbar_init(bar(BAR_ZK_EMPTY + i), 1);
    }
    for (int i = 0; i < kNZV; ++i) {
      mbar_init(bar(BAR_ZV_FULL + i), 1);
      mbar_init(bar(BAR_ZV_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(BAR_D_FULL + i), 1);
      mbar_init(bar(BAR_D_EMPTY + i), 4);
      mbar_init(bar(BAR_P_FULL + i), 4);
      mbar_init(bar(BAR_AT_FULL + i), 1);
      mbar_init(bar(BAR_AT_EMPTY + i), 4);
    }
    mbar_init(bar(BAR_EPI), 4);
    mbar_init(bar(BAR_TEARDOWN), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(base + L.tmem_slot, PS::kTmem);
    tmem_relinquish();
  }
  // P padding rows stay zero; q̃ rows of absent queries stay zero
  for (int i = threadIdx.x; i < 2 * kPB / 4; i += kThreads) reinterpret_cast<uint32_t*>(sbase + L.p)[i] = 0u;
  for (int i = threadIdx.x; i < nkc * kN * 32; i += kThreads) reinterpret_cast<uint32_t*>(sbase + L.qt)[i] = 0u;
  __syncthreads();
  // q̃ into the K-major swizzled B operand: row n = 8·jj + r of query jj, entry j
  for (int i = threadIdx.x; i < nq * 2 * kMaxG * r_k; i += kThreads) {
    const int n = i / r_k, j = i % r_k;
    const int jj = n >> 3, r = n & 7;
    const uint16_t* src = reinterpret_cast<const uint16_t*>(qt) +
                          ((((size_t)b * QN + jj) * gm.n + gi) * 2 * kMaxG + r) * a.r_k;   // rows a.r_k apart
    const int c = j / kChunk, kin = j % kChunk;
    *reinterpret_cast<uint16_t*>(sbase + L.qt + c * (kN * 128) + n * 128 + (((kin >> 3) ^ (n & 7)) << 4) +
                                 (kin & 7) * 2) = src[j];
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sbase + L.tmem_slot);

  if (warp == 0) {
    // ============================================================ producer (bulk copies)
    // The rings hold 160 KB, enough bytes in flight to cover HBM latency; a
    // bulk L2 prefetch of later pages on top of them measured slower here
    // (lines evicted before use: 1.44x the algorithmic DRAM bytes).
    if (lane == 0) {
      int zs = 0, vs = 0;
      uint32_t zph = 0, vph = 0;
      long long zk_issued = 0, zv_issued = 0;
      // z_v of a tile is needed only after its scores: stream it one tile behind
      // z_k, so the two rings fill in the order the MMAs consume them
      auto push_zv = [&](int k) -> bool {
        int pg = page_of(a, b, pg0 + k);
        if (pg < 0) pg = 0;   // reported with the keys
        const uint8_t* src = gm.zv[gi] + (size_t)pg * gm.v_page;
        for (int cb = 0; cb < 2 * NRV; ++cb) {
          if (!mbar_wait(bar(BAR_ZV_EMPTY + vs), vph ^ 1, abort_flag, st, 11)) return false;
          mbar_expect_tx(bar(BAR_ZV_FULL + vs), kStageBytes);
          bulk_load(base + L.zv + vs * kStageBytes, src + (size_t)cb * a.P * 128, kStageBytes, bar(BAR_ZV_FULL + vs));
          ++zv_issued;
          if (++vs == kNZV) { vs = 0; vph ^= 1; }
        }
        return true;
      };
      bool ok = true;
      for (int k = 0; k < ntiles && ok && !*abort_flag; ++k) {
        int pg = page_of(a, b, pg0 + k);
        if (pg < 0) {
          report(st, PALU_ERR_DEVICE_BOUNDS, 2000000 + b);
          pg = 0;   // keep the pipeline fed from a valid page; the status says the result is void
        }
        const uint8_t* src = gm.zk[gi] + (size_t)pg * gm.k_page;
        for (int c = 0; c < nkc; ++c) {
          if (!mbar_wait(bar(BAR_ZK_EMPTY + zs), zph ^ 1, abort_flag, st, 10)) { ok = false; break; }
          mbar_expect_tx(bar(BAR_ZK_FULL + zs), kStageBytes);
          bulk_load(base + L.zk + zs * kStageBytes, src + (size_t)c * kStageBytes, kStageBytes, bar(BAR_ZK_FULL + zs));
          ++zk_issued;
          if (++zs == kNZK) { zs = 0; zph ^= 1; }
        }
        if (ok && k >= 1 && k - 1 < nvt) ok = push_zv(k - 1);
      }
      if (ok && ntiles >= 1 && ntiles - 1 < nvt) push_zv(ntiles - 1);
      // after an abort, copies already issued still land in shared memory: wait for them
      drain_ring(bar(BAR_ZK_FULL), kNZK, zk_issued, st, 10);
      drain_ring(bar(BAR_ZV_FULL), kNZV, zv_issued, st, 11);
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      constexpr int kBf = ACT == PALU_BF16 ? 1 : 0;
      const uint32_t idesc_s = idesc_f16(kBf, 0, 0, kN, 128);    // z_k K-major, q̃ K-major
      const uint32_t idesc_pv = idesc_f16(kBf, 1, 0, kNP, 128);  // z_vᵀ MN-major, Pᵀ K-major
      int zs = 0, vs = 0;
      uint32_t zph = 0, vph = 0;
      // timeout-path test hook: first wait on a phase nothing completes before the teardown commit
      bool ok = a.stall_test == 0 || mbar_wait(bar(BAR_TEARDOWN), 0, abort_flag, st, 27);
      auto issue_pv = [&](int j) -> bool {
        const uint32_t a_tmem = tmem + PS::kAt + (uint32_t)(j & 1) * NRV * kNP;
        const uint32_t p_base = base + L.p + (uint32_t)(j & 1) * kPB;
        if (!mbar_wait(bar(BAR_P_FULL + (j & 1)), (j >> 1) & 1, abort_flag, st, 21)) return false;
        if (!mbar_wait(bar(BAR_AT_EMPTY + (j & 1)), ((j >> 1) & 1) ^ 1, abort_flag, st, 22)) return false;
        tc_fence_after();
        for (int mb = 0; mb < NRV; ++mb) {
          for (int cb = 0; cb < 2; ++cb)
            if (!mbar_wait(bar(BAR_ZV_FULL + vs + cb), vph, abort_flag, st, 23)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint64_t ad = sdesc(base + L.zv + vs * kStageBytes + kk * 16 * 128, kStageBytes, 1024, kSw128);
            const uint64_t bd = sdesc(p_base + (kk >> 2) * PS::kPRegion + (kk & 3) * 32, 16, 1024, kSw128);
            umma_f16(a_tmem + mb * kNP, ad, bd, idesc_pv, kk != 0);
          }
          umma_commit(bar(BAR_ZV_EMPTY + vs));
          umma_commit(bar(BAR_ZV_EMPTY + vs + 1));
          vs += 2;
          if (vs == kNZV) { vs = 0; vph ^= 1; }
        }
        umma_commit(bar(BAR_AT_FULL + (j & 1)));
        return true;
      };
      for (int k = 0; k < ntiles && ok; ++k) {
        const int slot = k & 1;
        if (!mbar_wait(bar(BAR_D_EMPTY + slot), ((k >> 1) & 1) ^ 1, abort_flag, st, 24)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)slot * kN;
        for (int c = 0; c < nkc; ++c) {
          if (!mbar_wait(bar(BAR_ZK_FULL + zs), zph, abort_flag, st, 25)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kChunk / 16; ++kk) {
            const uint64_t ad = sdesc(base + L.zk + zs * kStageBytes + kk * 32, 16, 1024, kSw128);
            const uint64_t bd = sdesc(base + L.qt + c * (kN * 128) + kk * 32, 16, 1024, kSw128);
            umma_f16(d_tmem, ad, bd, idesc_s, (c | kk) != 0);
          }
          umma_commit(bar(BAR_ZK_EMPTY + zs));
          if (++zs == kNZK) { zs = 0; zph ^= 1; }
        }
        if (!ok) break;
        umma_commit(bar(BAR_D_FULL + slot));
        // the previous tile's value MMA, once its P is written
        if (k >= 1 && k - 1 < nvt && !issue_pv(k - 1)) { ok = false; break; }
      }
      if (ok && ntiles >= 1 && ntiles - 1 < nvt) issue_pv(ntiles - 1);
      // drain, also after an abort: every MMA issued above completes before TMEM is released
      umma_commit(bar(BAR_TEARDOWN));
      mbar_drain(bar(BAR_TEARDOWN), 0, st, 26);
    }
  } else {
    // ============================================================ epilogue (warps 2-5)
    // One thread per token row (scores) and per latent row (value sums); the
    // (query, head) pairs of the pass are p = 4·jj + h.
    const int q4 = warp & 3;                 // TMEM lane quarter this warp may access
    const int row = q4 * 32 + lane;          // token row of the tile / latent row of aᵀ
    const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
    float* red = reinterpret_cast<float*>(sbase + L.red);
    uint32_t epi_phase = 0;
    auto ep_sync = [&](int where) -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_EPI));
      const bool r = mbar_wait(bar(BAR_EPI), epi_phase, abort_flag, st, where);
      epi_phase ^= 1;
      return r;
    };
    auto live = [&](int p) { return (p & 3) < gs && (p >> 2) < nq; };
    int qlim[QN];
#pragma unroll
    for (int jj = 0; jj < QN; ++jj) qlim[jj] = (a.causal && jj < nq) ? a.q_pos[(size_t)b * a.qpos_bstride + jj] : 0;
    float m_run[kPC], l_part[kPC], prev_scale[kPC];
    float acc[NRV][kPC];
#pragma unroll
    for (int p = 0; p < kPC; ++p) {
      m_run[p] = -INFINITY;
      l_part[p] = 0.f;
      prev_scale[p] = 0.f;
#pragma unroll
      for (int mb = 0; mb < NRV; ++mb) acc[mb][p] = 0.f;
    }
    auto fold_at = [&](int j) -> bool {
      if (!mbar_wait(bar(BAR_AT_FULL + (j & 1)), (j >> 1) & 1, abort_flag, st, 30)) return false;
      tc_fence_after();
#pragma unroll
      for (int mb = 0; mb < NRV; ++mb) {
        float v[kPC];
#pragma unroll
        for (int c = 0; c < kPC; c += 2)
          tmem_ld2(tmem + lane_addr + PS::kAt + (uint32_t)(j & 1) * NRV * kNP + mb * kNP + c, v + c);
        tmem_wait_ld();
#pragma unroll
        for (int p = 0; p < kPC; ++p)
          if (live(p)) acc[mb][p] = fmaf(acc[mb][p], prev_scale[p], v[p]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_AT_EMPTY + (j & 1)));
      return true;
    };
    bool ok = true;
    for (int k = 0; k < ntiles && ok; ++k) {
      const int slot = k & 1;
      const int t0 = (pg0 + k) * kTile;
      const bool in_seq = t0 + row < t_end;
      int pos = t0 + row;
      if (a.causal && a.pos_pool != nullptr) {
        const int pg = page_of(a, b, pg0 + k);
        pos = pg >= 0 ? a.pos_pool[(size_t)pg * a.P + row] : 0;
      }
      if (!mbar_wait(bar(BAR_D_FULL + slot), (k >> 1) & 1, abort_flag, st, 31)) { ok = false; break; }
      tc_fence_after();
      float d[8 * QN];
#pragma unroll
      for (int c = 0; c < 8 * QN; c += 2) tmem_ld2(tmem + lane_addr + slot * kN + c, d + c);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_D_EMPTY + slot));
      // the previous tile's latent sums are ready by now (its value MMA went
      // in behind this tile's scores)
      if (k >= 1 && !fold_at(k - 1)) { ok = false; break; }
      float sc[kPC];
      bool valid[QN];
#pragma unroll
      for (int jj = 0; jj < QN; ++jj)
        valid[jj] = in_seq && jj < nq && (!a.causal || pos <= qlim[jj]);   // causal among the new tokens
#pragma unroll
      for (int p = 0; p < kPC; ++p) {
        const int jj = p >> 2, h = p & 3;
        sc[p] = (valid[jj] && h < gs) ? d[8 * jj + h] + d[8 * jj + 4 + h] : -INFINITY;   // hi and lo parts of q̃
        float m = sc[p];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (lane == 0) red[((k & 1) * 4 + q4) * kPC + p] = m;
      }
      if (!ep_sync(33)) { ok = false; break; }
#pragma unroll
      for (int p = 0; p < kPC; ++p) {
        if (!live(p)) continue;
        const float* rr = red + (k & 1) * 4 * kPC + p;
        const float mt = fmaxf(fmaxf(rr[0], rr[kPC]), fmaxf(rr[2 * kPC], rr[3 * kPC]));
        const float m_new = fmaxf(m_run[p], mt);
        const float scale = m_new == -INFINITY ? 1.f : exp2f(m_run[p] - m_new);   // 1 while all masked
        const uint16_t pb = to_bits<ACT>(sc[p] != -INFINITY ? exp2f(sc[p] - m_new) : 0.f);
        *reinterpret_cast<uint16_t*>(sbase + L.p + slot * kPB + p_offset<QN>(p, row)) = pb;
        l_part[p] = fmaf(l_part[p], scale, from_bits<ACT>(pb));
        m_run[p] = m_new;
        prev_scale[p] = scale;
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_P_FULL + slot));
    }
    if (ok && ntiles > 0) {
      const int kl = ntiles - 1;
      if (!ragged_last) {
        ok = fold_at(kl);
      } else {
        // partial last page: a += Σ_{valid tokens} p · z_v on CUDA cores from the
        // valid rows only
        ok = ep_sync(34);   // every P entry of the tile is written
        const int t0 = (pg0 + kl) * kTile;
        const int nvalid = t_end - t0;
        const int pg = page_of(a, b, pg0 + kl);
        float at[NRV][kPC];
#pragma unroll
        for (int mb = 0; mb < NRV; ++mb)
#pragma unroll
          for (int p = 0; p < kPC; ++p) at[mb][p] = 0.f;
        if (pg >= 0) {
          const uint8_t* zv = gm.zv[gi] + (size_t)pg * gm.v_page;
          const uint8_t* pbuf = sbase + L.p + (kl & 1) * kPB;
          for (int t = 0; t < nvalid; ++t) {
            float z[NRV];
#pragma unroll
            for (int mb = 0; mb < NRV; ++mb) z[mb] = load_latent<ACT, ACT>(zv, t, a.P, nullptr, mb * 128 + row);
#pragma unroll
            for (int p = 0; p < kPC; ++p) {
              if (!live(p)) continue;
              const float pv = from_bits<ACT>(*reinterpret_cast<const uint16_t*>(pbuf + p_offset<QN>(p, t)));
#pragma unroll
              for (int mb = 0; mb < NRV; ++mb) at[mb][p] = fmaf(pv, z[mb], at[mb][p]);
            }
          }
        }
#pragma unroll
        for (int mb = 0; mb < NRV; ++mb)
#pragma unroll
          for (int p = 0; p < kPC; ++p) acc[mb][p] = fmaf(acc[mb][p], prev_scale[p], at[mb][p]);
      }
    }
    // l per pair: sum of the per-thread partials
    float* lred = reinterpret_cast<float*>(sbase + L.lred);
#pragma unroll
    for (int p = 0; p < kPC; ++p) {
      float v = l_part[p];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0) lred[q4 * kPC + p] = v;
    }
    ok = ep_sync(35) && ok;
    if (ok && !*abort_flag) {
      constexpr float kLn2 = 0.6931471805599453f;
#pragma unroll
      for (int p = 0; p < kPC; ++p) {
        if (!live(p)) continue;
        const int jj = p >> 2, h = p & 3;
        // partials of virtual sequence b·QN + jj (the combine maps it back)
        float* out = a.part + ((((size_t)b * QN + jj) * gm.n * gs + gi * gs + h) * a.S + s) * (a.r_v + 2);
        if (row == 0) {
          out[0] = ntiles > 0 ? m_run[p] * kLn2 : -INFINITY;
          out[1] = (lred[p] + lred[kPC + p]) + (lred[2 * kPC + p] + lred[3 * kPC + p]);
        }
#pragma unroll
        for (int mb = 0; mb < NRV; ++mb) out[2 + mb * 128 + row] = acc[mb][p];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, PS::kTmem);
  }
}

template <int ACT, int NRV, int QN>
cudaError_t launch_t(const DecodeArgs& a, cudaStream_t st) {
  void* qt = a.fused_q;
  const int vb = a.batch * QN;   // one folded query per (sequence, query slot of the pass)
  fold_query_kernel<ACT><<<dim3(a.gm.n, (a.r_k + 63) / 64, (vb + kFoldSeqs - 1) / kFoldSeqs), 256, 0, st>>>(a, QN, qt);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const Smem L = smem_layout<QN>(a.r_k);
  const size_t smem = L.total + 1024;
  auto kern = decode_fused_kernel<ACT, NRV, QN>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(a.S, a.gm.n, a.batch), kThreads, smem, st>>>(a, qt);
  count_launch();
  return cudaGetLastError();
}

// A pass serves exactly 1, 2 or 4 queries of every sequence (the caller splits
// a step's queries into such passes).
template <int ACT, int NRV>
cudaError_t launch_q(const DecodeArgs& a, cudaStream_t st) {
  if (a.qn == 1) return launch_t<ACT, NRV, 1>(a, st);
  if (a.qn == 2) return launch_t<ACT, NRV, 2>(a, st);
  if (a.qn == 4) return launch_t<ACT, NRV, 4>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace

bool fused_decode_supported(const palu_config* c) {
  if (c->rope_base != 0.f) return false;
  if (c->page_size != kTile || c->head_dim > 128 || c->head_dim % 8 != 0 || c->group_size > kMaxG) return false;
  if (c->act_dtype != PALU_F16 && c->act_dtype != PALU_BF16) return false;
  if (c->latent_dtype != c->act_dtype) return false;
  if (c->rank_k % 64 != 0 || c->rank_k > 512) return false;
  if (c->rank_v != 128 && c->rank_v != 256) return false;
  return smem_layout<kFusedMaxQueries>(c->rank_k).total + 1024 <= 227 * 1024;
}

int fused_queries_per_pass() { return kFusedMaxQueries; }

size_t fused_query_bytes(const palu_config* c, int batch) {
  const size_t G = (size_t)(c->num_heads / c->group_size);
  return (size_t)batch * G * 2 * kMaxG * c->rank_k * 2;
}

cudaError_t launch_decode_fused(const DecodeArgs& a, cudaStream_t st) {
  if (a.act == PALU_BF16) return a.r_v == 256 ? launch_q<PALU_BF16, 2>(a, st) : launch_q<PALU_BF16, 1>(a, st);
  return a.r_v == 256 ? launch_q<PALU_F16, 2>(a, st) : launch_q<PALU_F16, 1>(a, st);
}

}  // namespace palu
