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
//   warp 2  bulk-copy producer for z_v (its own ring, so neither stream waits on the other).
//   int4 latents: warps 12-15 dequantise z_k and warps 0, 2, 3 z_v into the
//           same rings instead (code × fp16 scale, rounded to the compute
//           dtype), so the MMAs below are the same for every latent dtype.
//   warp 1  MMA issuer: D[128 tok × 256] = z_k · B_k[:, 2 heads] into one of two
//           TMEM slots (kind::f16, fp32 accumulate); aᵀ[r_v × 16] = z_vᵀ · Pᵀ of
//           tile j into columns of tile j+1's slot that its epilogue has already
//           read, so no slot waits for a value round trip.
//   warps 4-11 epilogue, two warpgroups of one thread per token: tcgen05.ld the rebuilt keys,
//           rotate them (RoPE at the token's position), score against the
//           rotated query, online softmax (exp2), write P (bf16/fp16) for the
//           value MMA, fold the previous tile's aᵀ into running latent sums and
//           release the slot.
// Output: per (b, head, split) the partial (m, l, a[r_v]) the combine merges.
//
// This header holds the kernel template and its launcher; decode_tc.cu
// instantiates it for 16-bit latents and decode_tc_int4.cu for int4 latents,
// so that the code of one latent kind never moves the other's in its module.
#pragma once

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
constexpr int kChunk = 64;         // K chunk of z_k (elements) = one 128-byte column block of the page
constexpr int kRingStages = 5;     // z_k + z_v stages, either latent kind
constexpr uint32_t kZkSwz = 2u;    // 128-byte swizzle
constexpr uint32_t kZkSbo = 1024;  // bytes per 8-row swizzle atom
// Ring depths.  A z_v stage is one value-MMA operand of 128 latent entries × 64 tokens (two
// 64-entry column blocks of a token half), so stages are independent.  16-bit latents: 3 z_k
// stages, 2 z_v stages.  int4 latents convert codes locally, so the key ring needs less depth
// and the value ring gets a third stage: the value operand is converted ahead of its MMAs.
__host__ __device__ constexpr int zk_stages(bool int4) { return int4 ? 2 : 3; }
__host__ __device__ constexpr int zv_stages(bool int4) { return int4 ? 3 : 2; }
static_assert(zk_stages(false) + zv_stages(false) == kRingStages && zk_stages(true) + zv_stages(true) == kRingStages,
              "ring barrier slots");
constexpr int kPrefetch = 3;       // int4: pages of codes pulled into L2 ahead of the loads
constexpr int kBatch = 8;          // frequency pairs per TMEM round trip of the score pass
constexpr int kNB = 32 / kBatch;   // score batches per warpgroup and tile
// 16-bit latents: 12 warps (producers + MMA in warps 0-3, two epilogue warpgroups).
// int4 latents: 16 warps; the codes are converted to the compute dtype by warps 0, 2, 3
// (values) and 12-15 (keys), so the conversion keeps up with the tensor cores.
__host__ __device__ constexpr int threads_of(bool int4) { return int4 ? 512 : 384; }
// int4 register split (setmaxnreg): launched at 128 per thread (65,536 / 512), the two
// epilogue warpgroups take 168, warpgroup 0 (value conversion and the MMA thread) 104,
// the key converters 72: 2·168 + 104 + 72 = 4·128 (no spills in any role).
constexpr uint32_t kRegsLaunch = 128, kRegsEpi = 168, kRegsW0 = 104, kRegsKey = 72;
static_assert(2 * kRegsEpi + kRegsW0 + kRegsKey == 4 * kRegsLaunch, "register split");
constexpr int kZkBytes = kTile * kChunk * 2;   // bytes per z_k stage
constexpr int kZvBytes = 128 * 64 * 2;         // 16 KB: one 64-entry column block of a page (128 tokens)
constexpr int kPBytes = 16 * kTile * 2;        // 4 KB: 16 rows (heads, padded) × 128 tokens

struct Smem {
  // offsets in bytes from a 1024-aligned base
  uint32_t b, zk, zv, p, qr, psc, tb, omega, red, lred, bars, tmem_slot, abort, total;
};

// Every region but B_k (whose size follows the key rank) sits at a fixed offset,
// so the kernel's offsets are compile-time constants; B_k comes last.
__host__ __device__ inline Smem smem_layout(int r_k, bool int4) {
  Smem s{};
  uint32_t o = 0;
  s.zk = o;     o += zk_stages(int4) * kZkBytes;
  s.zv = o;     o += zv_stages(int4) * kZvBytes;
  s.p = o;      o += 2 * kPBytes;
  s.qr = o;     o += 3 * 128 * 4;                        // q'_i, q'_{i+64}, -q'_i per head pair row
  s.psc = o;    o += 2 * 2 * 128 * 4;
  s.tb = o;     o += 2 * 2 * 2 * 3 * 32 * 4;             // [warpgroup][tile parity][head][A|B|-A][32 freq]
  s.omega = o;  o += 64 * 8;
  s.red = o;    o += 2 * 4 * 2 * 4;
  s.lred = o;   o += 4 * 2 * 4;
  s.bars = o;   o += 32 * 8;
  s.tmem_slot = o; o += 16;
  s.abort = o;  o += 16;
  o = (o + 1023u) & ~1023u;                              // 128-byte-swizzle atoms: 1024-byte aligned
  s.b = o;      o += (uint32_t)r_k * 256 * 2;            // B_k for 2 heads
  s.total = o;
  return s;
}

// barrier indices
enum {
  BAR_B = 0,
  BAR_RINGS = 1,                     // z_k full, z_k empty, z_v full, z_v empty: one per stage (in the kernel)
  BAR_D_FULL = BAR_RINGS + 2 * kRingStages,  // 2
  BAR_D_EMPTY = BAR_D_FULL + 2,      // 2
  BAR_P_FULL = BAR_D_EMPTY + 2,      // 2
  BAR_AT_FULL = BAR_P_FULL + 2,      // 1
  BAR_TEARDOWN = BAR_AT_FULL + 1,
  BAR_EPI = BAR_TEARDOWN + 1,        // 2: per-warpgroup sync (4 warps), bounded
  BAR_QR = BAR_EPI + 2,              // rotated query staged
  BAR_XCH = BAR_QR + 1,              // 2: both warpgroups posted their cross-head partial scores
  BAR_MID = BAR_XCH + 2,             // the epilogue is halfway through a tile's score pass (one phase per tile)
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

// The producers read the table entry of a tile one tile before they use it
// (raw, checked at the use), so the dependent load never stalls the copies.
__device__ __forceinline__ int page_ahead(const DecodeArgs& a, int b, const TileRange& tr, int k) {
  return k < tr.ntiles ? a.page_table[(size_t)b * a.max_pages + tr.t_begin / kTile + k] : -1;
}
__device__ __forceinline__ bool page_valid(const DecodeArgs& a, int pg) { return pg >= 0 && pg < a.num_pages; }

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

// ---------------------------------------------------------------- int4 latents
// Sixteen bytes of a latent row = the 32 codes of one scale block.  Word m
// holds entries 8m..8m+7, entry e in bits 4e..4e+3 (two's complement; the even
// entry of each byte in its low nibble).  dequant8 turns one word into the 8
// values code × s rounded to the compute dtype, as one 16-byte unit of the
// shared-memory operand.
__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// PAIRED = false: the unit holds entries 0..7 in order.  PAIRED = true: the unit
// holds entries (0, 4, 1, 5, 2, 6, 3, 7), which saves the byte permutes where
// the consumer tracks the order (a row permutation of the value operand).
template <int ACT, bool PAIRED>
__device__ __forceinline__ uint4 dequant8(uint32_t x, uint16_t sbits) {
  uint4 o;
  if constexpr (ACT == PALU_F16) {
    // (code + 8) | 0x6400 is the half 1024 + code + 8: subtracting 1032 gives
    // the code exactly, and one half multiply rounds code × s once.
    const uint32_t r0 = (x & 0x000F000Fu) ^ 0x64086408u;           // entries 0, 4
    const uint32_t r1 = ((x >> 4) & 0x000F000Fu) ^ 0x64086408u;    // 1, 5
    const uint32_t r2 = ((x >> 8) & 0x000F000Fu) ^ 0x64086408u;    // 2, 6
    const uint32_t r3 = ((x >> 12) & 0x000F000Fu) ^ 0x64086408u;   // 3, 7
    const __half2 bias = bits_h2(0x64086408u);
    const __half sh = __ushort_as_half(sbits);
    const __half2 s2 = __halves2half2(sh, sh);
    auto cv = [&](uint32_t r) { return h2_bits(__hmul2(__hsub2(bits_h2(r), bias), s2)); };
    if constexpr (PAIRED) {
      o = make_uint4(cv(r0), cv(r1), cv(r2), cv(r3));
    } else {
      o = make_uint4(cv(__byte_perm(r0, r1, 0x5410)), cv(__byte_perm(r2, r3, 0x5410)),
                     cv(__byte_perm(r0, r1, 0x7632)), cv(__byte_perm(r2, r3, 0x7632)));
    }
  } else {
    // (code + 8) | 0x4B000000 is the float 2^23 + code + 8; code × s is exact
    // in fp32 and the pack rounds it to bf16 once.
    const float s = __half2float(__ushort_as_half(sbits));
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
      v[e] = (__int_as_float(((x >> (4 * e)) & 0xFu) ^ 0x4B000008u) - 8388616.0f) * s;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 h = PAIRED ? __floats2bfloat162_rn(v[e], v[e + 4]) : __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
      w[e] = *reinterpret_cast<uint32_t*>(&h);
    }
    o = make_uint4(w[0], w[1], w[2], w[3]);
  }
  return o;
}

// Latent entry held by row r of the value operand when its units are PAIRED.
__device__ __forceinline__ int paired_row(int r) { return (r & ~7) | ((r & 7) >> 1) | ((r & 1) << 2); }

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint16_t ld_shared_u16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Phase trace record (palu_debug_trace).
__device__ __forceinline__ void trace_record(const DecodeArgs& a, int ev, int k, long long t_start) {
  if (k >= a.trace_tiles) return;
  const size_t cta = ((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
  a.trace[(cta * 8 + ev) * a.trace_tiles + k] = clock64() - t_start;
}

// CONTIG: token positions are the cache slots (no position pool).  A separate
// instantiation keeps the per-token sincos path of explicit positions out of
// the score loop's instruction footprint.
template <int ACT, int NRV, int LAT, bool CONTIG>
__global__ void __launch_bounds__(threads_of(LAT == PALU_INT4), 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_bk, const __grid_constant__ DecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  // blockIdx.y: entry gi of the group map and head pair hp; the entry's key rank sets the layout
  const int gi = blockIdx.y / (a.gs / 2), hp = blockIdx.y % (a.gs / 2);
  const int r_k = a.gm.rk[gi];
  const Smem L = smem_layout(r_k, LAT == PALU_INT4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr bool kInt4 = LAT == PALU_INT4;
  constexpr int kNZK = zk_stages(kInt4);
  constexpr int kNVS = zv_stages(kInt4);
  constexpr int BAR_ZK_FULL = BAR_RINGS, BAR_ZK_EMPTY = BAR_ZK_FULL + kNZK;
  constexpr int BAR_ZV_FULL = BAR_ZK_EMPTY + kNZK, BAR_ZV_EMPTY = BAR_ZV_FULL + kNVS;
  constexpr int kThreads = threads_of(kInt4);
  static_assert(!kInt4 || NRV == 2, "int4 latents: r_v = 256");
  DevStatus* st = reinterpret_cast<DevStatus*>(a.status);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + L.abort);
  auto bar = [&](int i) { return base + L.bars + 8u * i; };

  const int b = blockIdx.z;
  const GroupMap& gm = a.gm;
  const int nkc = r_k / kChunk;
  const uint32_t k_blk_bytes = (uint32_t)a.P * (kInt4 ? r_k / 2 : 2 * r_k);   // this entry's block of a page
  const TileRange tr = tile_range(a, b, st, threadIdx.x == 0);
  const long long t_start = clock64();
  auto trace = [&](int ev, int k) {
    if (a.trace != nullptr) trace_record(a, ev, k, t_start);
  };

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    abort_init(abort_flag, a.wait_cycles);
    mbar_init(bar(BAR_B), 1);
    for (int i = 0; i < kNZK; ++i) {
      mbar_init(bar(BAR_ZK_FULL + i), kInt4 ? 4 : 1);   // int4: one arrival per converting warp
      mbar_init(bar(BAR_ZK_EMPTY + i), 1);
    }
    for (int i = 0; i < kNVS; ++i) {
      mbar_init(bar(BAR_ZV_FULL + i), kInt4 ? 3 : 1);
      mbar_init(bar(BAR_ZV_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(BAR_D_FULL + i), 1);
      mbar_init(bar(BAR_D_EMPTY + i), 8);
      mbar_init(bar(BAR_P_FULL + i), 8);
    }
    mbar_init(bar(BAR_AT_FULL), 1);
    mbar_init(bar(BAR_TEARDOWN), 1);
    mbar_init(bar(BAR_QR), 4);
    mbar_init(bar(BAR_MID), 8);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(BAR_EPI + i), 4);
      mbar_init(bar(BAR_XCH + i), 8);
    }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&tm_bk);
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

  if (warp == 0 && lane == 0) {
    mbar_expect_tx(bar(BAR_B), (uint32_t)r_k * 256 * 2);
    // 64-column blocks of B_k (MN-major, 128-byte swizzle), each in boxes of bk_box rows
    // int4 latents: the rows (latent entries) in the key converters' paired order, row
    // 8g + 2a + b of shared memory = row 8g + 4b + a of B_k (a 4-D view of B_k, see the launcher)
    for (int nb = 0; nb < 4; ++nb)
      for (int rb = 0; rb < r_k; rb += a.bk_box) {
        if constexpr (kInt4)
          tma_load_4d(base + L.b + (uint32_t)nb * r_k * 128 + rb * 128, &tm_bk, hp * 256 + nb * 64, 0, 0,
                      (gm.k_row0[gi] + rb) / 8, bar(BAR_B));
        else
          tma_load_2d(base + L.b + (uint32_t)nb * r_k * 128 + rb * 128, &tm_bk, hp * 256 + nb * 64,
                      gm.k_row0[gi] + rb, bar(BAR_B));
      }
  }
  // Roles.  int4 latents: each warpgroup first sets its share of the register file
  // (setmaxnreg, see kRegsLaunch), inside the branch whose code uses it.
  if (kInt4 && warp >= 12) {
    if constexpr (kInt4) setmaxnreg_dec<kRegsKey>();
    // ============================================================ int4 key codes (warps 12-15)
    // Chunk c of a tile = entries [64c, 64c + 64) of all 128 tokens, i.e. scale
    // blocks 2c and 2c+1 = 16-byte units 2c and 2c+1 of each token's row of codes.
    // Thread t takes both units of token t, loaded straight into registers three
    // chunks ahead of the conversion, while later pages are pulled into L2.  Entries
    // are written PAIRED (K position p of the operand holds entry paired_row(p)), which
    // saves byte permutes; B_k's rows are loaded in the same order, so the key MMA sums
    // the same products.
    const int t = threadIdx.x - 384;
    const int N = tr.ntiles * 4;
    struct Slot {
      uint4 raw[2];
      uint16_t sc[2];
    };
    auto prefetch_page = [&](int ppg) {
      if (t != 0 || !page_valid(a, ppg)) return;
      prefetch_l2(gm.zk[gi] + (size_t)ppg * gm.k_page, k_blk_bytes);
      prefetch_l2(gm.zks[gi] + (size_t)ppg * gm.ks_page, (uint32_t)(a.P * a.ks_row));
      prefetch_l2(gm.zv[gi] + (size_t)ppg * gm.v_page, (uint32_t)(a.P * a.v_row));
      prefetch_l2(gm.zvs[gi] + (size_t)ppg * gm.vs_page, (uint32_t)(a.P * a.vs_row));
    };
    // pg = the raw table entry of chunk n's tile, read a tile earlier
    auto issue = [&](int n, Slot& sl, int pg) {
      if (n >= N) return;
      if (!page_valid(a, pg)) {
        if ((n & 3) == 0 && t == 0) report(st, PALU_ERR_DEVICE_BOUNDS, 2000000 + b);
        pg = 0;   // keep the pipeline fed from a valid page; the status says the result is void
      }
      const uint8_t* row = gm.zk[gi] + (size_t)pg * gm.k_page + t * 128;
      const uint8_t* srow = gm.zks[gi] + (size_t)pg * gm.ks_page + (size_t)t * a.ks_row;
#pragma unroll
      for (int ub = 0; ub < 2; ++ub) {
        const int u = 2 * (n & 3) + ub;
        sl.raw[ub] = __ldg(reinterpret_cast<const uint4*>(row + ((u ^ (t & 7)) << 4)));
        sl.sc[ub] = __ldg(reinterpret_cast<const unsigned short*>(srow + 2 * u));
      }
    };
    int stage = 0;
    uint32_t phase = 0;
    auto consume = [&](int n, const Slot& sl) -> bool {
      if (n >= N) return true;
      if (!mbar_wait(bar(BAR_ZK_EMPTY + stage), phase ^ 1, abort_flag, st, 12)) return false;
      const uint32_t dst = base + L.zk + stage * kZkBytes + t * 128;
#pragma unroll
      for (int ub = 0; ub < 2; ++ub) {
        const uint32_t w[4] = {sl.raw[ub].x, sl.raw[ub].y, sl.raw[ub].z, sl.raw[ub].w};
#pragma unroll
        for (int m = 0; m < 4; ++m)
          st_shared_v4(dst + (((4 * ub + m) ^ (t & 7)) << 4), dequant8<ACT, true>(w[m], sl.sc[ub]));
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_ZK_FULL + stage));
      if (++stage == kNZK) { stage = 0; phase ^= 1; }
      return true;
    };
    Slot s0, s1, s2, s3;                               // after the shift: chunks n, n+1, n+2; s3 takes n+3
    for (int kk = 1; kk <= kPrefetch; ++kk) prefetch_page(page_ahead(a, b, tr, kk));
    int pg_k = page_ahead(a, b, tr, 0);                // tile k of chunk n
    int pg_k1 = page_ahead(a, b, tr, 1);               // tile k+1
    int pg_k2 = page_ahead(a, b, tr, 2);               // tile k+2, in flight
    int pf = page_ahead(a, b, tr, 1 + kPrefetch);      // tile k+1+kPrefetch, pulled into L2
    issue(0, s1, pg_k);
    issue(1, s2, pg_k);
    issue(2, s3, pg_k);
    // One load batch and one conversion per chunk: a single copy of the conversion
    // code keeps the kernel's instruction footprint small.  The register slots shift
    // down at the top of each iteration, before the next loads are issued, so a shift
    // never copies a slot whose loads went out in the same iteration (the copy would
    // wait for them).
#pragma unroll 1
    for (int n = 0; n < N && !*abort_flag; ++n) {
      const int c = n & 3;
      s0 = s1;
      s1 = s2;
      s2 = s3;
      if (c == 0 && n > 0) {
        pg_k = pg_k1;
        pg_k1 = pg_k2;
        pg_k2 = page_ahead(a, b, tr, (n >> 2) + 2);
      }
      issue(n + 3, s3, c == 0 ? pg_k : pg_k1);
      if (!consume(n, s0)) break;
      if (c == 0) {
        prefetch_page(pf);
        pf = page_ahead(a, b, tr, (n >> 2) + 2 + kPrefetch);
      }
    }
  } else if (warp >= 4) {
    if constexpr (kInt4) setmaxnreg_inc<kRegsEpi>();
    // ============================================================ epilogue (warps 4-11)
    // Two warpgroups split the 64 RoPE frequency pairs of every key (wg 0:
    // pairs [0, 32), wg 1: [32, 64)) for both heads, then each finishes one head.
    const int wg = (warp - 4) >> 2;
    const int q4 = warp & 3;                 // TMEM lane quarter this warp may access
    const int row = q4 * 32 + lane;          // token row of the tile / latent row of aᵀ
    const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
    float* qr = reinterpret_cast<float*>(sbase + L.qr);
    float* psc = reinterpret_cast<float*>(sbase + L.psc);   // [slot][head][128]
    const uint64_t* om = reinterpret_cast<const uint64_t*>(sbase + L.omega);
    const int head0 = gm.g[gi] * a.gs + hp * 2;   // model head of the pair's first head
    const int hl0 = gi * a.gs + hp * 2;           // the same head among this launch's heads
    constexpr float kLog2e = 1.4426950408889634f;
    // the 4 warps of one warpgroup meet here; a bounded wait (unlike bar.sync), so a thread that gave
    // up on a timed-out wait cannot strand the others.
    uint32_t epi_phase = 0;
    auto ep_sync = [&](int where) -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_EPI + wg));
      const bool r = mbar_wait(bar(BAR_EPI + wg), epi_phase, abort_flag, st, where);
      epi_phase ^= 1;
      return r;
    };
    // rotated query of both heads, scaled by log2(e)/sqrt(d_h) for exp2
    if (wg == 0) {
      const int hh = row >> 6, i = row & 63;
      using TA = typename Dt<ACT>::T;
      const TA* qh = reinterpret_cast<const TA*>(a.q) + (size_t)b * a.q_bstride + (size_t)(head0 + hh) * 128;
      const float x1 = Dt<ACT>::to_f(qh[i]), x2 = Dt<ACT>::to_f(qh[i + 64]);
      float c = 1.f, s = 0.f;
      if (a.rope) rope_cs_fast(a.q_pos[(size_t)b * a.qpos_bstride], a.omega[i], c, s);
      const float sc = a.sm_scale * kLog2e;
      const float qa = (x1 * c - x2 * s) * sc, qb = (x2 * c + x1 * s) * sc;
      qr[hh * 192 + i] = qa;
      qr[hh * 192 + 64 + i] = qb;
      qr[hh * 192 + 128 + i] = -qa;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_QR));
    }
    bool ok = mbar_wait(bar(BAR_QR), 0, abort_flag, st, 32);

    // Partial scores of both heads over this warpgroup's 32 frequency pairs i:
    //   score += c_i (q'_i k_i + q'_{i+64} k_{i+64}) + s_i (q'_{i+64} k_i - q'_i k_{i+64})
    // which is q'·k' with k' the key rotated by the token's angle (rotate-half).
    // Explicit positions take a sincos per token.  Contiguous positions (pos = t0 +
    // row): with (C, S) the cosine and sine at the tile start t0 and (c_r, s_r) those
    // at this thread's fixed offset `row`, angle addition turns the sum into
    //   score += c_r (k_i A_i + k_{i+64} B_i) + s_r (k_i B_i - k_{i+64} A_i),
    //   A_i = C q'_i + S q'_{i+64},  B_i = C q'_{i+64} - S q'_i,
    // i.e. the query rotated by the tile start, computed once per tile for the whole
    // warpgroup (double-buffered, published by the tile's softmax sync).  Math runs
    // on packed fp32 pairs (two frequencies at a time).
    constexpr bool contig = CONTIG;
    float* abuf = reinterpret_cast<float*>(sbase + L.tb) + wg * 384;   // [tile parity][head][A|B|-A][32]
    f2 crow[16], srow[16];
    if (contig) {
#pragma unroll
      for (int v = 0; v < 16; ++v) {
        float c0, s0, c1, s1;
        rope_cs_fast(row, om[wg * 32 + 2 * v], c0, s0);
        rope_cs_fast(row, om[wg * 32 + 2 * v + 1], c1, s1);
        crow[v] = f2_pack(c0, c1);
        srow[v] = f2_pack(s0, s1);
      }
    }
    // the query rotated by the start t0 of a tile, for this warpgroup's frequencies:
    // thread row < 64 takes frequency row mod 32 of head row / 32
    auto post_rotated_query = [&](int t0, int parity) {
      if (row >= 64) return;
      const int f = row & 31, hh = row >> 5;
      float c, sn;
      rope_cs_fast(t0, om[wg * 32 + f], c, sn);
      const float qa = qr[hh * 192 + wg * 32 + f], qb = qr[hh * 192 + 64 + wg * 32 + f];
      const float A = c * qa + sn * qb, B = c * qb - sn * qa;
      float* o = abuf + parity * 192 + hh * 96 + f;
      o[0] = A;
      o[32] = B;
      o[64] = -A;
    };
    auto half_scores = [&](int slot, int t0, int pos, float* part, auto&& mid) {
      const float* ab = abuf + ((t0 / kTile) & 1) * 192;
      f2 acc[2][2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) acc[hh][0] = acc[hh][1] = 0ull;
#pragma unroll
      for (int jj = 0; jj < kNB; ++jj) {
        mid(jj);   // halfway: signal that the first batches' columns are read
        const int i0 = wg * 32 + jj * kBatch;
        const uint32_t col = tmem + lane_addr + (uint32_t)slot * 256 + i0;
        // both heads' keys of these kBatch frequency pairs in one TMEM round trip
        float lo[2][kBatch], hi[2][kBatch];
        if constexpr (kBatch == 16) {
          tmem_ld16(col, lo[0]);
          tmem_ld16(col + 64, hi[0]);
          tmem_ld16(col + 128, lo[1]);
          tmem_ld16(col + 192, hi[1]);
        } else {
          tmem_ld8(col, lo[0]);
          tmem_ld8(col + 64, hi[0]);
          tmem_ld8(col + 128, lo[1]);
          tmem_ld8(col + 192, hi[1]);
        }
        tmem_wait_ld();
        if (contig) {
#pragma unroll
          for (int v4 = 0; v4 < kBatch / 4; ++v4) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const float* q = ab + hh * 96 + jj * kBatch + 4 * v4;
              const float4 A4 = *reinterpret_cast<const float4*>(q);
              const float4 B4 = *reinterpret_cast<const float4*>(q + 32);
              const float4 N4 = *reinterpret_cast<const float4*>(q + 64);
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int v = v4 * 2 + e, vr = jj * (kBatch / 2) + v;
                const f2 A2 = e ? f2_pack(A4.z, A4.w) : f2_pack(A4.x, A4.y);
                const f2 B2 = e ? f2_pack(B4.z, B4.w) : f2_pack(B4.x, B4.y);
                const f2 N2 = e ? f2_pack(N4.z, N4.w) : f2_pack(N4.x, N4.y);
                const f2 lo2 = f2_pack(lo[hh][2 * v], lo[hh][2 * v + 1]);
                const f2 hi2 = f2_pack(hi[hh][2 * v], hi[hh][2 * v + 1]);
                const f2 u = f2_fma(hi2, B2, f2_mul(lo2, A2));   // k_i A_i + k_{i+64} B_i
                const f2 w = f2_fma(lo2, B2, f2_mul(hi2, N2));   // k_i B_i - k_{i+64} A_i
                acc[hh][e] = f2_fma(crow[vr], u, acc[hh][e]);
                acc[hh][e] = f2_fma(srow[vr], w, acc[hh][e]);
              }
            }
          }
          continue;
        }
#pragma unroll
        for (int v4 = 0; v4 < kBatch / 4; ++v4) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int v = v4 * 2 + e;
            f2 cs, sn;
            {
              // explicit positions: a sincos per token
              float c0, s0, c1, s1;
              rope_cs_fast(pos, om[i0 + 2 * v], c0, s0);
              rope_cs_fast(pos, om[i0 + 2 * v + 1], c1, s1);
              cs = f2_pack(c0, c1);
              sn = f2_pack(s0, s1);
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const float* qh = qr + hh * 192 + i0 + 4 * v4 + 2 * e;
              const f2 a2 = *reinterpret_cast<const f2*>(qh);
              const f2 b2 = *reinterpret_cast<const f2*>(qh + 64);
              const f2 n2 = *reinterpret_cast<const f2*>(qh + 128);
              const f2 lo2 = f2_pack(lo[hh][2 * v], lo[hh][2 * v + 1]);
              const f2 hi2 = f2_pack(hi[hh][2 * v], hi[hh][2 * v + 1]);
              const f2 x = f2_fma(b2, hi2, f2_mul(a2, lo2));     // q'_i k_i + q'_{i+64} k_{i+64}
              const f2 y = f2_fma(b2, lo2, f2_mul(n2, hi2));     // q'_{i+64} k_i - q'_i k_{i+64}
              acc[hh][e] = f2_fma(cs, x, acc[hh][e]);
              acc[hh][e] = f2_fma(sn, y, acc[hh][e]);
            }
          }
        }
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float a0, a1, a2, a3;
        f2_unpack(acc[hh][0], a0, a1);
        f2_unpack(acc[hh][1], a2, a3);
        part[hh] = (a0 + a1) + (a2 + a3);
      }
    };

    {
      // Each warpgroup owns one head of the pair (hw = wg) for the softmax, P,
      // the latent value sums and the output; the partial scores of the other
      // head go across in shared memory.
      const int hw = wg;
      // latent entry of TMEM lane `row` of aᵀ (int4: the value operand's units are PAIRED)
      const int vrow = kInt4 ? paired_row(row) : row;
      float m_run = -INFINITY, l_part = 0.f, prev_scale = 0.f;
      float acc[NRV];
#pragma unroll
      for (int mb = 0; mb < NRV; ++mb) acc[mb] = 0.f;
      float* red = reinterpret_cast<float*>(sbase + L.red);

      // The value sums of tile j sit in the TMEM slot of tile j + 1 (columns [32·mb, +16),
      // column hw of each block for this head); fold them into the running sums.
      auto fold_at = [&](int j, float scale) -> bool {
        if (!mbar_wait(bar(BAR_AT_FULL), j & 1, abort_flag, st, 30)) return false;
        tc_fence_after();
        const uint32_t sb = (uint32_t)((j + 1) & 1) * 256;
#pragma unroll
        for (int mb = 0; mb < NRV; ++mb) {
          const float v = tmem_ld1(tmem + lane_addr + sb + mb * 32 + hw);
          tmem_wait_ld();
          acc[mb] = fmaf(acc[mb], scale, v);
        }
        return true;
      };

      const int nv_tiles = tr.ntiles - (tr.ragged_last ? 1 : 0);   // tiles whose value sums are MMAs
      // causal bound (several queries per step): tokens after the query's position are masked
      const int qlim = a.causal ? a.q_pos[(size_t)b * a.qpos_bstride] : 0;
      if (contig && tr.ntiles > 0) {
        post_rotated_query(tr.t_begin, (tr.t_begin / kTile) & 1);
        ok = ep_sync(37) && ok;
      }
      for (int k = 0; k < tr.ntiles && ok; ++k) {
        const int t0 = tr.t_begin + k * kTile;
        int pos = t0 + row;
        if (a.pos_pool != nullptr) {
          const int pg = page_of(a, b, t0 / kTile);
          pos = pg >= 0 ? a.pos_pool[(size_t)pg * a.P + row] : 0;
        }
        const bool valid = t0 + row < tr.t_end && (!a.causal || pos <= qlim);
        const int slot = k & 1;
        if (!mbar_wait(bar(BAR_D_FULL + slot), (k >> 1) & 1, abort_flag, st, 31)) { ok = false; break; }
        tc_fence_after();
        if (row == 0 && wg == 0) trace(3, k);
        float part[2];
        // Halfway through the pass (score batches 0 and 1 read) the columns where the
        // previous tile's value MMA writes are dead: tell the MMA thread.
        half_scores(slot, t0, pos, part, [&](int jj) {
          if (jj != kNB / 2) return;
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BAR_MID));
        });
        // the next tile's rotated query; the tile-max sync below publishes it
        if (contig) post_rotated_query(t0 + kTile, ((t0 / kTile) + 1) & 1);
        psc[(slot * 2 + (1 - hw)) * 128 + row] = part[1 - hw];
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_XCH + slot));
        if (!mbar_wait(bar(BAR_XCH + slot), (k >> 1) & 1, abort_flag, st, 36)) { ok = false; break; }
        const float sfull = part[hw] + psc[(slot * 2 + hw) * 128 + row];
        if (row == 0 && wg == 0) trace(4, k);
        // tile max of this head across the 128 tokens
        const float sc = valid ? sfull : -INFINITY;
        float m = sc;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (lane == 0) red[(k & 1) * 8 + wg * 4 + q4] = m;
        if (!ep_sync(33)) { ok = false; break; }
        const float* rr = red + (k & 1) * 8 + wg * 4;
        const float mt = fmaxf(fmaxf(rr[0], rr[1]), fmaxf(rr[2], rr[3]));
        const float m_new = fmaxf(m_run, mt);
        // 0 on the first tile; 1 while every token so far is masked
        const float scale = m_new == -INFINITY ? 1.f : exp2f(m_run - m_new);
        const uint16_t pb = to_bits<ACT>(valid ? exp2f(sc - m_new) : 0.f);
        *reinterpret_cast<uint16_t*>(sbase + L.p + slot * kPBytes + p_offset(hw, row)) = pb;
        l_part = fmaf(l_part, scale, from_bits<ACT>(pb));
        m_run = m_new;
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_P_FULL + slot));
        if (row == 0 && wg == 0) trace(5, k);
        // the previous tile's value sums (written into this slot), then release the slot
        if (k >= 1 && k - 1 < nv_tiles && !fold_at(k - 1, prev_scale)) { ok = false; break; }
        prev_scale = scale;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_D_EMPTY + slot));
      }

      if (ok && tr.ntiles > 0) {
        const int kl = tr.ntiles - 1;
        if (!tr.ragged_last) {
          ok = fold_at(kl, prev_scale);
        } else {
          // partial last page: a += Σ_{valid tokens} p · z_v on CUDA cores,
          // reading only the valid rows (the rest of the page is never touched)
          ok = ep_sync(34);   // every P entry of this head is written
          const int t0 = tr.t_begin + kl * kTile;
          const int nvalid = tr.t_end - t0;
          const int pg = page_of(a, b, t0 / kTile);
          float at[NRV];
#pragma unroll
          for (int mb = 0; mb < NRV; ++mb) at[mb] = 0.f;
          if (pg >= 0) {
            const uint8_t* zv = gm.zv[gi] + (size_t)pg * gm.v_page;
            const uint8_t* zvs = kInt4 ? gm.zvs[gi] + (size_t)pg * gm.vs_page : nullptr;
            const uint8_t* pbuf = sbase + L.p + (kl & 1) * kPBytes;
            for (int t = 0; t < nvalid; ++t) {
              const float pv = from_bits<ACT>(*reinterpret_cast<const uint16_t*>(pbuf + p_offset(hw, t)));
              const uint8_t* srow = kInt4 ? zvs + (size_t)t * a.vs_row : nullptr;
#pragma unroll
              for (int mb = 0; mb < NRV; ++mb)
                at[mb] = fmaf(pv, load_latent<LAT, ACT>(zv, t, a.P, srow, mb * 128 + vrow), at[mb]);
            }
          }
#pragma unroll
          for (int mb = 0; mb < NRV; ++mb) acc[mb] = fmaf(acc[mb], prev_scale, at[mb]);
        }
      }

      // l: sum of the per-thread partials of this head
      float* lred = reinterpret_cast<float*>(sbase + L.lred);
      float v = l_part;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0) lred[wg * 4 + q4] = v;
      ok = ep_sync(35) && ok;
      if (ok && !*abort_flag) {
        constexpr float kLn2 = 0.6931471805599453f;
        float* out = a.part + (((size_t)b * gm.n * a.gs + hl0 + hw) * a.S + blockIdx.x) * (a.r_v + 2);
        if (row == 0) {
          out[0] = tr.ntiles > 0 ? m_run * kLn2 : -INFINITY;
          out[1] = (lred[wg * 4 + 0] + lred[wg * 4 + 1]) + (lred[wg * 4 + 2] + lred[wg * 4 + 3]);
        }
#pragma unroll
        for (int mb = 0; mb < NRV; ++mb) out[2 + mb * 128 + vrow] = acc[mb];
      }
    }
  } else {
    // warps 0-3
    if constexpr (kInt4) setmaxnreg_dec<kRegsW0>();
    if (kInt4 && warp != 1) {
      // ============================================================ int4 value codes (warps 0, 2, 3)
      // Ring stage s of a tile (s = 2mb + th) = entries [128mb, +128) of tokens
      // [64th, +64) = 16-byte units 4mb .. 4mb+3 of those tokens' rows of codes: 256
      // (token, unit) items, dealt to the 96 threads round-robin (item i: token
      // 64th + i mod 64, unit 4mb + i / 64) and loaded straight into registers two
      // stages ahead of the conversion.  Unit j = i / 64 lands in the stage's 64-entry
      // block j / 2 (8 KB apart), its 32 entries written PAIRED: row r of the value
      // operand holds entry paired_row(r).
      const int vt = (warp == 0 ? 0 : warp == 2 ? 32 : 64) + lane;
      const int nv_tiles = tr.ntiles - (tr.ragged_last ? 1 : 0);
      constexpr int kSPT = 2 * NRV;                      // ring stages per tile
      const int N = nv_tiles * kSPT;
      struct Slot {
        uint4 raw[3];
        uint16_t sc[3];
      };
      // pg = the raw table entry of stage n's tile, read a tile earlier
      auto issue = [&](int n, Slot& sl, int pg) {
        if (n >= N) return;
        if (!page_valid(a, pg)) pg = 0;   // reported by the key converters
        const uint8_t* blk = gm.zv[gi] + (size_t)pg * gm.v_page;
        const uint8_t* sblk = gm.zvs[gi] + (size_t)pg * gm.vs_page;
        const int s = n % kSPT, mb = s >> 1, th = s & 1;
  #pragma unroll
        for (int j = 0; j < 3; ++j) {
          const int i = vt + 96 * j;
          if (i < 256) {
            const int t = 64 * th + (i & 63), u = 4 * mb + (i >> 6);
            sl.raw[j] = __ldg(reinterpret_cast<const uint4*>(blk + t * 128 + ((u ^ (t & 7)) << 4)));
            sl.sc[j] = __ldg(reinterpret_cast<const unsigned short*>(sblk + (size_t)t * a.vs_row + 2 * u));
          }
        }
      };
      int stage = 0;
      uint32_t phase = 0;
      auto consume = [&](int n, const Slot& sl) -> bool {
        if (n >= N) return true;
        if (!mbar_wait(bar(BAR_ZV_EMPTY + stage), phase ^ 1, abort_flag, st, 13)) return false;
        if (vt == 0 && n % kSPT == 0) trace(6, n / kSPT);
        const uint32_t dst = base + L.zv + stage * kZvBytes;
  #pragma unroll
        for (int j = 0; j < 3; ++j) {
          const int i = vt + 96 * j;
          if (i < 256) {
            const int tr64 = i & 63, blk = (i >> 7), ub = (i >> 6) & 1;   // token row, entry block, unit
            const uint32_t w[4] = {sl.raw[j].x, sl.raw[j].y, sl.raw[j].z, sl.raw[j].w};
            const uint32_t row = dst + blk * (kZvBytes / 2) + tr64 * 128;
  #pragma unroll
            for (int m = 0; m < 4; ++m)
              st_shared_v4(row + (((4 * ub + m) ^ (tr64 & 7)) << 4), dequant8<ACT, true>(w[m], sl.sc[j]));
          }
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_ZV_FULL + stage));
        if (++stage == kNVS) { stage = 0; phase ^= 1; }
        return true;
      };
      Slot s0, s1, s2;                                   // after the shift: stages n, n+1; s2 takes n+2
      int pg_k = page_ahead(a, b, tr, 0);                // tile k of stage n
      int pg_k1 = page_ahead(a, b, tr, 1);               // tile k+1
      int pg_k2 = page_ahead(a, b, tr, 2);               // tile k+2, in flight
      issue(0, s1, pg_k);
      issue(1, s2, pg_k);
      // as for the keys: the slots shift before the next loads go out
  #pragma unroll 1
      for (int n = 0; n < N && !*abort_flag; ++n) {
        s0 = s1;
        s1 = s2;
        if (n % kSPT == 0 && n > 0) {
          pg_k = pg_k1;
          pg_k1 = pg_k2;
          pg_k2 = page_ahead(a, b, tr, n / kSPT + 2);
        }
        issue(n + 2, s2, (n + 2) / kSPT == n / kSPT ? pg_k : pg_k1);
        if (!consume(n, s0)) break;
      }
    } else if (warp == 0) {
      // ============================================================ z_k producer (bulk copies)
      if (lane == 0) {
        int stage = 0;
        uint32_t phase = 0;
        // No bulk L2 prefetch of later pages here: with the bulk copies of the two
        // head-pair CTAs of a group in flight, a prefetch 3 or 6 pages ahead left the
        // copy latency unchanged and the call 2-3 % slower.
        int pg_next = page_ahead(a, b, tr, 0);
        long long issued = 0;
        for (int k = 0; k < tr.ntiles && !*abort_flag; ++k) {
          int pg = pg_next;
          pg_next = page_ahead(a, b, tr, k + 1);   // in flight during this tile's copies
          if (!page_valid(a, pg)) {
            report(st, PALU_ERR_DEVICE_BOUNDS, 2000000 + b);
            pg = 0;   // keep the pipeline fed from a valid page; the status says the result is void
          }
          // one (page, group) block is the shared-memory image of the tile: each
          // 128-byte column block (64 latent entries of all 128 tokens) is one copy
          const uint8_t* src = gm.zk[gi] + (size_t)pg * gm.k_page;
          for (int c = 0; c < nkc; ++c) {
            if (!mbar_wait(bar(BAR_ZK_EMPTY + stage), phase ^ 1, abort_flag, st, 10)) break;
            mbar_expect_tx(bar(BAR_ZK_FULL + stage), kZkBytes);
            bulk_load(base + L.zk + stage * kZkBytes, src + (size_t)c * kZkBytes, kZkBytes, bar(BAR_ZK_FULL + stage));
            ++issued;
            if (++stage == kNZK) { stage = 0; phase ^= 1; }
          }
        }
        drain_ring(bar(BAR_ZK_FULL), kNZK, issued, st, 10);
      }
    } else if (warp == 2) {
      // ============================================================ z_v producer (bulk copies)
      if (lane == 0) {
        int stage = 0;
        uint32_t phase = 0;
        int pg_next = page_ahead(a, b, tr, 0);
        long long issued = 0;
        for (int k = 0; k < tr.ntiles && !*abort_flag; ++k) {
          if (tr.ragged_last && k == tr.ntiles - 1) break;    // CUDA-core value sum for a partial page
          int pg = pg_next;
          pg_next = page_ahead(a, b, tr, k + 1);   // in flight during this tile's copies
          if (!page_valid(a, pg)) pg = 0;   // reported by the z_k producer
          const uint8_t* src = gm.zv[gi] + (size_t)pg * gm.v_page;
          // one 16 KB copy per 128-byte column block of the page (64 latent entries of all
          // 128 tokens); the two stages of the ring are the two 64-entry halves of one
          // value-MMA operand (whole blocks copied faster than token halves of 8 KB)
          for (int cb = 0; cb < 2 * NRV; ++cb) {
            if (!mbar_wait(bar(BAR_ZV_EMPTY + stage), phase ^ 1, abort_flag, st, 11)) break;
            mbar_expect_tx(bar(BAR_ZV_FULL + stage), kZvBytes);
            bulk_load(base + L.zv + stage * kZvBytes, src + (size_t)cb * a.P * 128, kZvBytes,
                      bar(BAR_ZV_FULL + stage));
            if (cb == 0) trace(6, k);
            ++issued;
            if (++stage == kNVS) { stage = 0; phase ^= 1; }
          }
        }
        drain_ring(bar(BAR_ZV_FULL), kNVS, issued, st, 11);
      }
    } else if (warp == 1) {
      // ============================================================ MMA issuer
      if (lane == 0) {
        constexpr int kBf = ACT == PALU_BF16 ? 1 : 0;
        const uint32_t idesc_d = idesc_f16(kBf, 0, 1, 256, 128);    // z_k K-major, B_k MN-major
        const uint32_t idesc_pv = idesc_f16(kBf, 1, 0, 16, 128);    // z_vᵀ MN-major, Pᵀ K-major
        const uint32_t b_lbo = (uint32_t)r_k * 128;                  // bytes between 64-column blocks of B
        int zs = 0;
        uint32_t zph = 0, vph = 0;
        // timeout-path test hook: first wait on a phase nothing completes before the teardown commit
        bool ok = a.stall_test == 0 || mbar_wait(bar(BAR_TEARDOWN), 0, abort_flag, st, 26);
        ok = ok && mbar_wait(bar(BAR_B), 0, abort_flag, st, 20);
        const int nv_tiles = tr.ntiles - (tr.ragged_last ? 1 : 0);   // tiles whose value sums run here
        int pv_next = 0;       // next tile whose value MMA is not issued yet
        int pv_s = 0;          // next operand of that value MMA: block mb = pv_s / 2 (int4: token half pv_s % 2)
        int vs = 0;            // int4: z_v ring stage of that operand
        int zv_seen = -1;      // last tile whose value latents were seen in shared memory (trace)

        // The value MMA of tile j, aᵀ[128 entries × 16] per block mb = z_vᵀ · Pᵀ, goes into
        // columns [32·mb, +16) of the TMEM slot of tile j + 1: columns whose keys that
        // tile's epilogue has read by the middle of its score pass (BAR_MID), so the value
        // round trip never holds a slot back from the next key MMA.  The last tile's value
        // MMA goes into the other slot once it is free.  Its gate (besides P and z_v):
        auto pv_gate = [&](int j) -> bool {
          if (j + 1 < tr.ntiles) return mbar_test_wait(bar(BAR_MID), (uint32_t)((j + 1) & 1));
          const int u = j + 1;
          return mbar_test_wait(bar(BAR_D_EMPTY + (u & 1)), (uint32_t)(((u >> 1) & 1) ^ 1));
        };
        // The next stage of the pending value MMA can go?  (Phases cannot alias: the
        // epilogue cannot pass tile j + 1 before the value sums of tile j are folded.)
        // int4: one ring stage per operand (mb, th); 16-bit latents: the two stages of the
        // ring hold the two 64-entry halves of operand mb over all 128 tokens.
        auto pv_ready = [&]() -> bool {
          if (pv_next >= nv_tiles) return false;
          if constexpr (kInt4) {
            if (!mbar_test_wait(bar(BAR_ZV_FULL + vs), vph)) return false;
          } else {
            if (!(mbar_test_wait(bar(BAR_ZV_FULL + 0), vph) && mbar_test_wait(bar(BAR_ZV_FULL + 1), vph)))
              return false;
          }
          if (pv_s == 0 && zv_seen != pv_next) {
            zv_seen = pv_next;
            trace(7, pv_next);
          }
          return pv_s > 0 || (mbar_test_wait(bar(BAR_P_FULL + (pv_next & 1)), (uint32_t)((pv_next >> 1) & 1)) &&
                              pv_gate(pv_next));
        };
        // One value-MMA operand into block mb of the value sums.  int4: stage (mb, th) =
        // latent entries [128mb, +128) (two 64-entry blocks 8 KB apart) × tokens [64th, +64),
        // against the matching half of Pᵀ.  16-bit latents: the two ring stages (64 entries
        // of all 128 tokens each) against all of Pᵀ.
        auto issue_pv_block = [&]() {
          const int j = pv_next;
          tc_fence_after();
          const uint32_t p_base = base + L.p + (uint32_t)(j & 1) * kPBytes;
          if constexpr (kInt4) {
            const int mb = pv_s >> 1, th = pv_s & 1;
            const uint32_t a_tmem = tmem + (uint32_t)((j + 1) & 1) * 256 + (uint32_t)mb * 32;
            const uint32_t z_base = base + L.zv + (uint32_t)vs * kZvBytes;
  #pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              // rows = latent entries, K = 16 tokens of the half
              const uint64_t ad = sdesc(z_base + kk * 16 * 128, kZvBytes / 2, 1024, kSw128);
              const uint64_t bd = sdesc(p_base + th * 2048 + kk * 32, 16, 1024, kSw128);
              umma_f16(a_tmem, ad, bd, idesc_pv, (th | kk) != 0);
            }
            umma_commit(bar(BAR_ZV_EMPTY + vs));
            if (++vs == kNVS) { vs = 0; vph ^= 1; }
            ++pv_s;
          } else {
            static_assert(kInt4 || zv_stages(false) == 2, "one value MMA operand = the two ring stages");
            const uint32_t a_tmem = tmem + (uint32_t)((j + 1) & 1) * 256 + (uint32_t)(pv_s >> 1) * 32;
  #pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk) {
              // rows = latent entries (two 64-entry blocks, one per stage), K = tokens
              const uint64_t ad = sdesc(base + L.zv + kk * 16 * 128, kZvBytes, 1024, kSw128);
              const uint64_t bd = sdesc(p_base + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024, kSw128);
              umma_f16(a_tmem, ad, bd, idesc_pv, kk != 0);
            }
            umma_commit(bar(BAR_ZV_EMPTY + 0));
            umma_commit(bar(BAR_ZV_EMPTY + 1));
            vph ^= 1;
            pv_s += 2;
          }
          if (pv_s == 2 * NRV) {
            umma_commit(bar(BAR_AT_FULL));
            trace(2, j);
            ++pv_next;
            pv_s = 0;
          }
        };
        // Wait for a barrier phase; meanwhile issue every value-MMA block whose operands
        // and gate are in (the epilogue's slot releases depend on them).  Bounded.
        auto poll_wait = [&](uint32_t b, uint32_t parity, int where) -> bool {
          const long long t0 = clock64();
          while (true) {
            if (mbar_test_wait(b, parity)) return true;
            if (pv_ready()) {
              issue_pv_block();
              continue;
            }
            if (*abort_flag) return false;
            __nanosleep(64);   // leave the issue slots of this SM partition to the epilogue warps
            if (clock64() - t0 > wait_limit(abort_flag)) {
              report(st, PALU_ERR_DEVICE_TIMEOUT, where);
              *abort_flag = 1;
              return false;
            }
          }
        };

        for (int k = 0; k < tr.ntiles && ok; ++k) {
          const int slot = k & 1;
          if (!poll_wait(bar(BAR_D_EMPTY + slot), ((k >> 1) & 1) ^ 1, 23)) { ok = false; break; }
          tc_fence_after();
          trace(0, k);
          const uint32_t d_tmem = tmem + (uint32_t)slot * 256;
          for (int c = 0; c < nkc; ++c) {
            if (!poll_wait(bar(BAR_ZK_FULL + zs), zph, 24)) { ok = false; break; }
            tc_fence_after();
            const uint32_t zk_addr = base + L.zk + zs * kZkBytes;
            const uint32_t b_addr = base + L.b + (uint32_t)c * kChunk * 128;
  #pragma unroll
            for (int kk = 0; kk < kChunk / 16; ++kk) {
              const uint64_t ad = sdesc(zk_addr + kk * 32, 16, kZkSbo, kZkSwz);
              const uint64_t bd = sdesc(b_addr + kk * 16 * 128, b_lbo, 1024, kSw128);
              umma_f16(d_tmem, ad, bd, idesc_d, (c | kk) != 0);
            }
            umma_commit(bar(BAR_ZK_EMPTY + zs));
            if (++zs == kNZK) { zs = 0; zph ^= 1; }
          }
          if (!ok) break;
          umma_commit(bar(BAR_D_FULL + slot));
          trace(1, k);
        }
        // the value MMAs still pending (the last tiles'), each once its operands are in
        if (ok) {
          const long long t0 = clock64();
          while (pv_next < nv_tiles) {
            if (pv_ready()) {
              issue_pv_block();
              continue;
            }
            if (*abort_flag) break;
            __nanosleep(64);
            if (clock64() - t0 > wait_limit(abort_flag)) {
              report(st, PALU_ERR_DEVICE_TIMEOUT, 21);
              *abort_flag = 1;
              break;
            }
          }
        }
        // drain, also after an abort: every MMA issued above has completed before
        // TMEM is released, and the B_k load has landed before the CTA exits
        umma_commit(bar(BAR_TEARDOWN));
        mbar_drain(bar(BAR_TEARDOWN), 0, st, 25);
        mbar_drain(bar(BAR_B), 0, st, 20);
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
                 uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  (void)elt_bytes;
  CUresult r = fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// B_k (row-major [rows][W], 16-bit) as a 4-D map for the paired row order: dims (innermost
// first) columns, b (stride 4 rows), a (stride 1 row), g (stride 8 rows); boxes of 64
// columns × 2 × 4 × box_rows/8.
bool make_map_bk_paired(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, uint64_t W, uint64_t rows,
                        uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const uint64_t rb = W * 2;   // bytes per row
  cuuint64_t dims[4] = {W, 2, 4, rows / 8};
  cuuint64_t strides[3] = {4 * rb, rb, 8 * rb};
  cuuint32_t box[4] = {64, 2, 4, box_rows / 8};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, dt, 4, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int ACT, int NRV, int LAT>
cudaError_t launch_t(const DecodeArgs& a, cudaStream_t st) {
  const CUtensorMapDataType dt = ACT == PALU_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap tm_bk;
  if (a.bk_box <= 0 || a.bk_box > 256 || a.bk_box % 64 != 0) return cudaErrorInvalidValue;
  if constexpr (LAT == PALU_INT4) {
    // B_k viewed as [rows / 8][a: 4][b: 2][W] with the b dimension traversed before a, so a
    // box lands row 8g + 4b + a of B_k at row 8g + 2a + b of shared memory: the paired
    // order the key converters write the latent entries in
    if (a.bk_rows % 8 != 0 || !make_map_bk_paired(&tm_bk, a.Bk, dt, a.W, (uint64_t)a.bk_rows, a.bk_box))
      return cudaErrorInvalidValue;
  } else if (!make_map_2d(&tm_bk, a.Bk, dt, 2, a.W, (uint64_t)a.bk_rows, (uint64_t)a.W * 2, 64, a.bk_box,
                          CU_TENSOR_MAP_SWIZZLE_128B)) {
    return cudaErrorInvalidValue;
  }
  const Smem L = smem_layout(a.r_k, LAT == PALU_INT4);
  const size_t smem = L.total + 1024;
  auto kern = a.pos_pool == nullptr ? decode_tc_kernel<ACT, NRV, LAT, true> : decode_tc_kernel<ACT, NRV, LAT, false>;
  DecodeArgs args = a;
  const TraceSetting ts = trace_setting();
  const size_t ctas = (size_t)a.S * a.gm.n * (a.gs / 2) * a.batch;
  if (ts.buffer != nullptr && ctas * 8 * (size_t)ts.tiles * 8 <= ts.bytes) {
    args.trace = static_cast<long long*>(ts.buffer);
    args.trace_tiles = ts.tiles;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if constexpr (LAT == PALU_INT4) {
    // The warpgroups' setmaxnreg split adds up to exactly the registers of a launch at
    // kRegsLaunch per thread; launched with fewer, the epilogue's increase could never
    // be granted.  Refuse to launch a build whose kernel is not at that count.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != (int)kRegsLaunch) return cudaErrorInvalidConfiguration;
  }
  dim3 grid(a.S, a.gm.n * (a.gs / 2), a.batch);
  kern<<<grid, threads_of(LAT == PALU_INT4), smem, st>>>(tm_bk, args);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

}  // namespace palu
