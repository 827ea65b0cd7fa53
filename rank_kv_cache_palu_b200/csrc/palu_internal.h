// Internal interface between the C-ABI layer (palu_abi.cu) and the kernel
// launchers.  Host-side only; not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "palu.h"

namespace palu {

constexpr int kMaxHalfDim = 64;  // head_dim <= 128
constexpr int kMaxGroups = 64;   // head groups per layer

// Where the head groups a launch covers keep their latents.  All groups of a
// launch share one rank pair (r_k, r_v); a layer whose groups have different
// ranks runs one launch per rank pair.  With one pool for all groups (equal
// ranks), group g's block of page pg starts at pool + (pg·G + g)·P·row; with a
// pool per group, at pool_g + pg·P·row_g.  Either way: base[g] + pg·page.
struct GroupMap {
  int n;                                // groups this launch covers
  uint16_t g[kMaxGroups];               // model group of entry i (heads g·gs .. g·gs + gs − 1)
  const uint8_t* zk[kMaxGroups];        // per model group: block of page 0
  const uint8_t* zv[kMaxGroups];
  const uint8_t* zks[kMaxGroups];       // int4 scale rows (NULL otherwise)
  const uint8_t* zvs[kMaxGroups];
  long long k_page, v_page, ks_page, vs_page;   // bytes from one page's block to the next
  uint16_t k_row0[kMaxGroups];          // first row of the group in B_k (= first column in A_k)
  uint16_t v_row0[kMaxGroups];          // same for B_v / A_v
  uint16_t rk[kMaxGroups];              // key rank of the entry (decode launches may mix key ranks;
                                        // the launch's r_k is their maximum, r_v is shared)
};

// Everything a decode launch needs, already validated.
struct DecodeArgs {
  int H, d_h, gs, G, W, r_k, r_v, P;
  int batch, max_pages, num_pages, S;
  int act, lat;        // palu_dtype values
  int rope;            // 0: RoPE off
  float sm_scale;      // 1/sqrt(d_h)
  const void* q;
  const int32_t* q_pos;
  // Per-sequence strides of q / q_pos / out / lse (elements): H·d_h, 1, H·d_h,
  // H for one query per sequence; Q times that when a step holds Q queries
  // and one launch serves one of them.
  long long q_bstride, o_bstride;
  int qpos_bstride, lse_bstride;
  int causal;          // 1: a token counts only if its position <= the query's position
  int qn;              // queries of each sequence this launch serves (the fused kernel takes
                       // several per pass; their partials sit at virtual sequence b·qn + j)
  GroupMap gm;
  const int32_t* pos_pool;
  const int32_t* page_table;
  const int32_t* seq_lens;
  const void* Bk;      // [bk_rows][W]: group entry i's rows start at gm.k_row0[i]
  const void* Bv;      // [bv_rows][W]
  int bk_rows, bv_rows;
  int bk_box;          // rows per tensor-map box of B_k: the key rank when every entry has it, else 64
  void* out;
  float* lse;
  float* part;         // [batch·qn][gm.n·gs][S][r_v + 2] float32, heads in group-map order
  void* fused_q;       // fused (no-RoPE) path: folded queries [batch·qn][gm.n][8][r_k], act dtype
  void* status;        // DevStatus*
  long long k_row, v_row, ks_row, vs_row;  // bytes per latent / scale row
  uint64_t omega[kMaxHalfDim];             // RoPE frequencies as 64-bit fixed-point turns
  long long* trace;                        // phase trace (palu_debug_trace) or NULL
  int trace_tiles;
  long long wait_cycles;                   // bound of every wait in the tensor-core kernels (SM cycles)
  int stall_test;                          // timeout-path test: the MMA thread first waits on a phase
                                           // that nothing completes, so the launch times out
};

// Phase-trace buffer set by palu_debug_trace (NULL: off).
struct TraceSetting {
  void* buffer;
  size_t bytes;
  int tiles;
};
TraceSetting trace_setting();

struct CompressArgs {
  int n, d_model, G, r_k, r_v, P, num_pages;
  int act, lat;
  const void* x;
  const void* Ak;
  const void* Av;
  const int32_t* slots;
  const int32_t* positions;
  GroupMap gm;         // the groups of this launch; A column offsets in k_row0 / v_row0
  long long a_kcols, a_vcols;   // columns of A_k / A_v (row strides in elements)
  // Output columns of this launch, key side: entry i owns [kcol[i], kcol[i + 1]) (its rank
  // wide; ranks may differ between entries), kcol[gm.n] = ncols_k; likewise the value side.
  int ncols_k, ncols_v;
  uint16_t kcol[kMaxGroups + 1], vcol[kMaxGroups + 1];
  int32_t* pos_pool;
  void* status;
  float* scratch;  // workspace past the status header
  size_t scratch_bytes;
  long long k_row, v_row, ks_row, vs_row;
  long long wait_cycles;   // as in DecodeArgs
  int stall_test;
};

// Wait bound and stall switch of the timeout-path test (palu_debug_timeout_test).
struct TimeoutTest {
  long long wait_cycles;   // <= 0: the default (about a second)
  int stall;
};
TimeoutTest timeout_test_setting();

// CUDA-core kernels (any supported dtype; the only path for float32).
cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t st);
cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t st);
cudaError_t launch_compress_simt(const CompressArgs& a, cudaStream_t st);

// Counts kernel launches (palu_kernel_launches); call once per launch.
void count_launch(int n = 1);

// Row bytes of the pools for a config.
inline long long latent_row_bytes(int lat, int r) {
  switch (lat) {
    case PALU_F32: return 4LL * r;
    case PALU_F16:
    case PALU_BF16: return 2LL * r;
    case PALU_INT4: return r / 2;
  }
  return 0;
}
inline long long scale_row_bytes(int lat, int r) {
  if (lat != PALU_INT4) return 0;
  long long b = 2LL * (r / 32);
  return (b + 15) / 16 * 16;
}

}  // namespace palu
