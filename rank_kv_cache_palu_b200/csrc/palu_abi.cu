// C-ABI layer of libpalu.so: argument checks, workspace layout, kernel choice.
// Every entry point validates synchronously and returns a palu_status; nothing
// throws or aborts across the ABI.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "palu_common.cuh"
#include "palu_internal.h"
#include "palu_tc.h"

namespace palu {
static std::atomic<unsigned long long> g_launches{0};
static TraceSetting g_trace{nullptr, 0, 0};
TraceSetting trace_setting() { return g_trace; }
static TimeoutTest g_timeout_test{0, 0};
TimeoutTest timeout_test_setting() { return g_timeout_test; }
void count_launch(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }
}  // namespace palu

namespace {

thread_local char g_cuda_err[256] = "";

palu_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return PALU_OK;
  snprintf(g_cuda_err, sizeof(g_cuda_err), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return PALU_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

palu_status check_config(const palu_config* c) {
  if (c == nullptr) return PALU_ERR_INVALID_ARG;
  if (c->num_heads <= 0 || c->head_dim <= 0 || c->group_size <= 0 || c->rank_k <= 0 ||
      c->rank_v <= 0 || c->page_size <= 0)
    return PALU_ERR_INVALID_ARG;
  if (c->num_heads % c->group_size != 0) return PALU_ERR_INVALID_ARG;
  if (c->head_dim % 2 != 0) return PALU_ERR_INVALID_ARG;
  if (!(c->rope_base >= 0.f) || isinf(c->rope_base)) return PALU_ERR_INVALID_ARG;
  if (c->act_dtype < PALU_F32 || c->act_dtype > PALU_BF16) return PALU_ERR_INVALID_ARG;
  if (c->latent_dtype < PALU_F32 || c->latent_dtype > PALU_INT4) return PALU_ERR_INVALID_ARG;
  // supported pairs: latent == act, or int4 latents with a 16-bit compute dtype
  const bool pair_ok = (c->latent_dtype == c->act_dtype) ||
                       (c->latent_dtype == PALU_INT4 && c->act_dtype != PALU_F32);
  if (!pair_ok) return PALU_ERR_UNSUPPORTED;
  if (c->head_dim > 2 * palu::kMaxHalfDim) return PALU_ERR_UNSUPPORTED;
  if (c->rank_k > 512 || c->rank_v > 512) return PALU_ERR_UNSUPPORTED;
  if (c->num_heads / c->group_size > palu::kMaxGroups) return PALU_ERR_UNSUPPORTED;
  // latent rows are whole 128-byte column blocks (the swizzled page layout)
  if (palu::latent_row_bytes(c->latent_dtype, c->rank_k) % 128 != 0 ||
      palu::latent_row_bytes(c->latent_dtype, c->rank_v) % 128 != 0)
    return PALU_ERR_ALIGNMENT;
  if (c->page_size % 8 != 0) return PALU_ERR_ALIGNMENT;
  return PALU_OK;
}

void fill_omega(const palu_config* c, uint64_t* omega) {
  const int half = c->head_dim / 2;
  const long double two_pi = 6.283185307179586476925286766559005768L;
  for (int i = 0; i < palu::kMaxHalfDim; ++i) {
    if (i >= half || c->rope_base == 0.f) {
      omega[i] = 0;
      continue;
    }
    const long double theta = powl((long double)c->rope_base, -2.0L * i / c->head_dim);
    const long double turns = theta / two_pi;  // < 1
    omega[i] = (uint64_t)llroundl(ldexpl(turns, 64));  // 64-bit fixed-point fraction (< 2^62)
  }
}

constexpr size_t kStatusBytes = sizeof(palu::DevStatus);
constexpr int kMaxQueries = PALU_MAX_QUERIES;

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Queries of each sequence one launch serves: the fused kernel takes passes
// of 4, 2 or 1 queries; the other kernels one query per launch.
int pass_queries(int kind, int remaining) {
  if (kind != 3) return 1;
  const int m = palu::fused_queries_per_pass();
  return remaining >= m ? m : remaining >= 2 ? 2 : 1;
}

int auto_splits(const palu_config* c, int batch, int max_pages, int kind, int qn = 1) {
  const int sms = 148;
  const long long groups = (long long)batch * (c->num_heads / c->group_size);
  const long long units = kind == 3   ? groups
                          : kind == 2 ? groups * palu::tc_head_blocks(c)
                                      : (long long)batch * c->num_heads;
  if (units <= 0) return 1;
  if (kind == 1) {
    // CUDA-core kernel: enough CTAs for ~4 waves of one CTA per SM
    long long S = (4LL * sms + units - 1) / units;
    if (S > max_pages) S = max_pages;
    return (int)(S < 1 ? 1 : S > 256 ? 256 : S);
  }
  // Tensor-core kernels hold one CTA per SM and every CTA of a launch walks about
  // the same number of pages, so the launch takes ceil(CTAs / SMs) rounds of
  // (pages per split + a start-up of ~2 pages); with several queries per pass the
  // combine adds about a page per split and query (measured: 4 queries per pass at
  // 16 x 16k ran best at 4 splits, one query at 8).  Take the split count that minimises that (the
  // smallest on ties), sized for the longest possible sequence (max_pages), from one full round
  // of CTAs up -- or from the largest count that fits one round when that keeps >= 90 % of the
  // SMs busy (a round a few SMs short beats two rounds when the units do not divide the SM count).
  long long S0 = (sms + units - 1) / units;
  if (units * (sms / units) * 10 >= 9LL * sms) S0 = sms / units;
  if (S0 > max_pages) S0 = max_pages;
  if (S0 < 1) S0 = 1;
  long long best_S = S0, best_t = -1;
  for (long long S = S0; S <= max_pages && S <= 64; ++S) {
    const long long rounds = (units * S + sms - 1) / sms;
    const long long t = rounds * ((max_pages + S - 1) / S + 2) + (qn > 1 ? S * qn : 0);
    if (best_t < 0 || t < best_t) {
      best_t = t;
      best_S = S;
    }
  }
  return (int)best_S;
}

int kernel_kind(const palu_config* c) {
  if (check_config(c) != PALU_OK) return 0;
  if (palu::fused_decode_supported(c)) return 3;
  if (palu::tc_decode_supported(c)) return 2;
  return 1;
}

// The split count a call runs (num_splits = 0: automatic); qn = queries per pass.
int run_S(const palu_config* c, int kind, int batch, int max_pages, int num_splits, int qn = 1) {
  return num_splits == 0 ? auto_splits(c, batch, max_pages, kind, qn) : num_splits;
}

// One layer's head groups and where their latents live.  Group g has its own
// rank pair (r_k,g, r_v,g) — one pair for all groups unless the caller gives a
// rank per group.  A page of the K pool holds every group's block back to back,
// group g's at byte Σ_{g'<g} P·row_k,g' (likewise V and the int4 scale pools);
// B_k stacks the groups' [r_k,g × W] blocks, so group g's rows start at
// Σ_{g'<g} r_k,g', and A_k's columns follow the same order.  With one rank pair
// this is the layout pool[page][g][P rows].  Groups with equal rank pairs form
// a class, which one launch of the compress kernel serves.  The decode kernels
// take a key rank per group: one launch serves every group with the same value
// rank and kernel family (a decode set).
struct Layer {
  palu_config cfg;   // model shape and dtypes (rank fields: see rk / rv)
  int G;
  int rk[palu::kMaxGroups], rv[palu::kMaxGroups];
  long long k_off[palu::kMaxGroups], v_off[palu::kMaxGroups];
  long long ks_off[palu::kMaxGroups], vs_off[palu::kMaxGroups];
  long long k_page, v_page, ks_page, vs_page;   // bytes per page of each pool
  int k_row0[palu::kMaxGroups], v_row0[palu::kMaxGroups];
  int bk_rows, bv_rows;                         // Σ r_k,g and Σ r_v,g
  int nclass;
  int cls[palu::kMaxGroups];                    // class of each group
  int crk[palu::kMaxGroups], crv[palu::kMaxGroups], cn[palu::kMaxGroups];
  int nset;
  int dset[palu::kMaxGroups];                   // decode set of each group
  int srk[palu::kMaxGroups], srv[palu::kMaxGroups], sn[palu::kMaxGroups];   // max key rank, value rank, groups
};

palu_status make_layer(const palu_config* cfg, const int32_t* ranks_k, const int32_t* ranks_v, Layer* L) {
  if (cfg == nullptr || (ranks_k == nullptr) != (ranks_v == nullptr)) return PALU_ERR_INVALID_ARG;
  // the shape checks, with group 0's ranks standing in for cfg's when ranks are given
  palu_config c0 = *cfg;
  if (ranks_k != nullptr) {
    c0.rank_k = ranks_k[0];
    c0.rank_v = ranks_v[0];
  }
  palu_status s = check_config(&c0);
  if (s != PALU_OK) return s;
  L->cfg = *cfg;
  const int G = cfg->num_heads / cfg->group_size;
  const long long P = cfg->page_size;
  const int lat = cfg->latent_dtype;
  L->G = G;
  L->nclass = 0;
  long long ko = 0, vo = 0, kso = 0, vso = 0;
  int kr = 0, vr = 0;
  for (int g = 0; g < G; ++g) {
    palu_config c = *cfg;
    c.rank_k = ranks_k ? ranks_k[g] : cfg->rank_k;
    c.rank_v = ranks_v ? ranks_v[g] : cfg->rank_v;
    s = check_config(&c);
    if (s != PALU_OK) return s;
    L->rk[g] = c.rank_k;
    L->rv[g] = c.rank_v;
    L->k_off[g] = ko;
    L->v_off[g] = vo;
    L->ks_off[g] = kso;
    L->vs_off[g] = vso;
    ko += P * palu::latent_row_bytes(lat, c.rank_k);
    vo += P * palu::latent_row_bytes(lat, c.rank_v);
    kso += P * palu::scale_row_bytes(lat, c.rank_k);
    vso += P * palu::scale_row_bytes(lat, c.rank_v);
    L->k_row0[g] = kr;
    L->v_row0[g] = vr;
    kr += c.rank_k;
    vr += c.rank_v;
    int k = 0;
    while (k < L->nclass && !(L->crk[k] == c.rank_k && L->crv[k] == c.rank_v)) ++k;
    if (k == L->nclass) {
      L->crk[k] = c.rank_k;
      L->crv[k] = c.rank_v;
      L->cn[k] = 0;
      ++L->nclass;
    }
    L->cls[g] = k;
    ++L->cn[k];
  }
  L->k_page = ko;
  L->v_page = vo;
  L->ks_page = kso;
  L->vs_page = vso;
  L->bk_rows = kr;
  L->bv_rows = vr;
  // decode sets: one value rank and one kernel family (the family's limits grow
  // with the key rank, so the set's largest key rank is supported as well)
  L->nset = 0;
  for (int g = 0; g < G; ++g) {
    palu_config c = *cfg;
    c.rank_k = L->rk[g];
    c.rank_v = L->rv[g];
    const int kind = kernel_kind(&c);
    int k = 0;
    while (k < L->nset) {
      palu_config d = *cfg;
      d.rank_k = L->srk[k];
      d.rank_v = L->srv[k];
      if (L->srv[k] == c.rank_v && kernel_kind(&d) == kind) break;
      ++k;
    }
    if (k == L->nset) {
      L->srk[k] = c.rank_k;
      L->srv[k] = c.rank_v;
      L->sn[k] = 0;
      ++L->nset;
    }
    if (c.rank_k > L->srk[k]) L->srk[k] = c.rank_k;
    L->dset[g] = k;
    ++L->sn[k];
  }
  return PALU_OK;
}

// The config one compress class's launch sees: its groups and its ranks.
palu_config class_cfg(const Layer& L, int c) {
  palu_config x = L.cfg;
  x.num_heads = L.cn[c] * L.cfg.group_size;
  x.rank_k = L.crk[c];
  x.rank_v = L.crv[c];
  return x;
}

// The config one decode set's launches see: its groups, its largest key rank, its value rank.
palu_config set_cfg(const Layer& L, int k) {
  palu_config x = L.cfg;
  x.num_heads = L.sn[k] * L.cfg.group_size;
  x.rank_k = L.srk[k];
  x.rank_v = L.srv[k];
  return x;
}

// Group map of the groups g with part[g] == c (a decode set), or of every group (part NULL).
void build_map(const Layer& L, const int* part, int c, const void* zk, const void* zv, const void* zks,
               const void* zvs, palu::GroupMap& m) {
  auto at = [](const void* pool, long long off) {
    return pool == nullptr ? nullptr : static_cast<const uint8_t*>(pool) + off;
  };
  m.n = 0;
  m.k_page = L.k_page;
  m.v_page = L.v_page;
  m.ks_page = L.ks_page;
  m.vs_page = L.vs_page;
  for (int g = 0; g < L.G; ++g) {
    if (part != nullptr && part[g] != c) continue;
    const int i = m.n++;
    m.g[i] = (uint16_t)g;
    m.zk[i] = at(zk, L.k_off[g]);
    m.zv[i] = at(zv, L.v_off[g]);
    m.zks[i] = at(zks, L.ks_off[g]);
    m.zvs[i] = at(zvs, L.vs_off[g]);
    m.k_row0[i] = (uint16_t)L.k_row0[g];
    m.v_row0[i] = (uint16_t)L.v_row0[g];
    m.rk[i] = (uint16_t)L.rk[g];
  }
}

// Decode workspace: the status word, then the partials of the largest decode
// set ([vb][heads][S][r_v + 2] float32, vb = sequence × query slot of a pass),
// then the folded queries of the largest fused-kernel set.  Sets run one after
// another on the stream, so they share both regions.
size_t decode_workspace(const Layer& L, int batch, int Q, int max_pages, int num_splits, size_t* fused_off) {
  size_t part = 0, fq = 0;
  for (int c = 0; c < L.nset; ++c) {
    const palu_config cc = set_cfg(L, c);
    const int kind = kernel_kind(&cc);
    const int S = run_S(&cc, kind, batch, max_pages, num_splits, pass_queries(kind, Q));
    const int vb = batch * pass_queries(kind, Q);
    const size_t pc = align256((size_t)vb * cc.num_heads * S * (cc.rank_v + 2) * sizeof(float));
    if (pc > part) part = pc;
    if (kind == 3) {
      const size_t f = align256(palu::fused_query_bytes(&cc, vb));
      if (f > fq) fq = f;
    }
  }
  if (fused_off) *fused_off = kStatusBytes + part;
  return kStatusBytes + part + fq;
}

// The compress kernels take every group of the layer in one launch (output
// columns follow the groups' ranks); the tensor-core kernel serves the layer
// when it serves each group's rank pair.
bool compress_tc_ok(const Layer& L, int n_tokens, int d_model) {
  for (int c = 0; c < L.nclass; ++c) {
    const palu_config cc = class_cfg(L, c);
    if (!palu::tc_compress_supported(&cc, n_tokens, d_model)) return false;
  }
  return true;
}

size_t compress_workspace(const Layer& L, int n_tokens, int d_model) {
  if (!compress_tc_ok(L, n_tokens, d_model)) return kStatusBytes;
  const palu_config c0 = class_cfg(L, 0);
  return kStatusBytes + palu::tc_compress_scratch_bytes(&c0, n_tokens, d_model, L.bk_rows, L.bv_rows);
}

palu_status compress_layer(const Layer& L, int n_tokens, int d_model, const void* x, const void* A_k,
                           const void* A_v, const int32_t* slot_mapping, const int32_t* positions, void* zk_pool,
                           void* zv_pool, void* zk_scales, void* zv_scales, int32_t* pos_pool, int num_pages,
                           void* workspace, size_t workspace_bytes, palu_stream_t stream) {
  const palu_config* cfg = &L.cfg;
  if (n_tokens < 0 || d_model <= 0 || num_pages < 0) return PALU_ERR_INVALID_ARG;
  if (d_model % 64 != 0) return PALU_ERR_UNSUPPORTED;
  if (workspace == nullptr || workspace_bytes < compress_workspace(L, n_tokens, d_model)) return PALU_ERR_WORKSPACE;
  if (n_tokens == 0) return PALU_OK;
  if (!x || !A_k || !A_v || !slot_mapping || !zk_pool || !zv_pool) return PALU_ERR_INVALID_ARG;
  const bool int4 = cfg->latent_dtype == PALU_INT4;
  if (int4 && (!zk_scales || !zv_scales)) return PALU_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(A_k) || !aligned16(A_v) || !aligned16(zk_pool) ||
      !aligned16(zv_pool) || (int4 && (!aligned16(zk_scales) || !aligned16(zv_scales))) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return PALU_ERR_ALIGNMENT;

  palu::CompressArgs a{};
  a.n = n_tokens;
  a.d_model = d_model;
  a.G = L.G;
  a.P = cfg->page_size;
  a.num_pages = num_pages;
  a.act = cfg->act_dtype;
  a.lat = cfg->latent_dtype;
  a.x = x;
  a.Ak = A_k;
  a.Av = A_v;
  a.slots = slot_mapping;
  a.pos_pool = pos_pool;
  a.status = workspace;
  a.scratch = reinterpret_cast<float*>(static_cast<char*>(workspace) + kStatusBytes);
  a.scratch_bytes = workspace_bytes - kStatusBytes;
  a.wait_cycles = palu::timeout_test_setting().wait_cycles;
  a.stall_test = palu::timeout_test_setting().stall;
  a.a_kcols = L.bk_rows;
  a.a_vcols = L.bv_rows;
  a.positions = positions;
  // every group in one launch: output column c of the key side is column c of A_k
  // (the groups' columns follow each other in order), owned by group col_entry(kcol, G, c)
  build_map(L, nullptr, 0, zk_pool, zv_pool, zk_scales, zv_scales, a.gm);
  a.ncols_k = L.bk_rows;
  a.ncols_v = L.bv_rows;
  for (int g = 0; g <= L.G; ++g) {
    a.kcol[g] = (uint16_t)(g < L.G ? L.k_row0[g] : L.bk_rows);
    a.vcol[g] = (uint16_t)(g < L.G ? L.v_row0[g] : L.bv_rows);
  }
  a.r_k = a.r_v = 0;   // per group: see kcol / vcol
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e = compress_tc_ok(L, n_tokens, d_model) ? palu::launch_compress_tc(a, st)
                                                             : palu::launch_compress_simt(a, st);
  if (e != cudaSuccess) return cuda_status(e);
  return PALU_OK;
}

// One decode step for Q queries per sequence (Q = 1: palu_decode_attn).  Each
// decode set runs its split kernel and combine over its own groups; within a
// set, passes of queries run one after another on the stream, sharing the
// workspace.  With Q > 1 a query attends only to the tokens at or before its
// own position.
palu_status decode_layer(const Layer& L, int batch, int Q, const void* q, const int32_t* q_pos,
                         const void* zk_pool, const void* zv_pool, const void* zk_scales, const void* zv_scales,
                         const int32_t* pos_pool, const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                         int num_pages, const void* B_k, const void* B_v, void* out, float* lse, void* workspace,
                         size_t workspace_bytes, int num_splits, palu_stream_t stream) {
  const palu_config* cfg = &L.cfg;
  if (batch < 0 || max_pages <= 0 || num_pages < 0 || num_splits < 0 || Q < 1 || Q > kMaxQueries)
    return PALU_ERR_INVALID_ARG;
  if (num_splits > max_pages) return PALU_ERR_INVALID_ARG;
  size_t fused_off = 0;
  const size_t need = decode_workspace(L, batch, Q, max_pages, num_splits, &fused_off);
  if (workspace == nullptr || workspace_bytes < need) return PALU_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PALU_ERR_ALIGNMENT;
  if (batch == 0) return PALU_OK;
  if (!q || !q_pos || !zk_pool || !zv_pool || !page_table || !seq_lens || !B_k || !B_v || !out)
    return PALU_ERR_INVALID_ARG;
  const bool int4 = cfg->latent_dtype == PALU_INT4;
  if (int4 && (!zk_scales || !zv_scales)) return PALU_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(zk_pool) || !aligned16(zv_pool) || !aligned16(B_k) ||
      !aligned16(B_v) || (int4 && (!aligned16(zk_scales) || !aligned16(zv_scales))))
    return PALU_ERR_ALIGNMENT;

  palu::DecodeArgs a{};
  a.H = cfg->num_heads;
  a.d_h = cfg->head_dim;
  a.gs = cfg->group_size;
  a.G = L.G;
  a.W = cfg->group_size * cfg->head_dim;
  a.P = cfg->page_size;
  a.batch = batch;
  a.max_pages = max_pages;
  a.num_pages = num_pages;
  a.act = cfg->act_dtype;
  a.lat = cfg->latent_dtype;
  a.rope = cfg->rope_base != 0.f;
  a.sm_scale = (float)(1.0 / sqrt((double)cfg->head_dim));
  a.pos_pool = pos_pool;
  a.page_table = page_table;
  a.seq_lens = seq_lens;
  a.Bk = B_k;
  a.Bv = B_v;
  a.bk_rows = L.bk_rows;
  a.bv_rows = L.bv_rows;
  a.status = workspace;
  a.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + kStatusBytes);
  a.fused_q = static_cast<char*>(workspace) + fused_off;
  a.wait_cycles = palu::timeout_test_setting().wait_cycles;
  a.stall_test = palu::timeout_test_setting().stall;
  fill_omega(cfg, a.omega);

  const long long qrow = (long long)a.H * a.d_h;       // one query's elements per sequence
  const size_t elt = cfg->act_dtype == PALU_F32 ? 4 : 2;
  if (Q > 1 && (qrow * (long long)elt) % 16 != 0) return PALU_ERR_ALIGNMENT;
  a.q_bstride = Q * qrow;
  a.o_bstride = Q * qrow;
  a.qpos_bstride = Q;
  a.lse_bstride = Q * a.H;
  a.causal = Q > 1;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  for (int c = 0; c < L.nset; ++c) {
    const palu_config cc = set_cfg(L, c);
    const int kind = kernel_kind(&cc);
    a.S = run_S(&cc, kind, batch, max_pages, num_splits, pass_queries(kind, Q));
    a.r_k = cc.rank_k;
    a.r_v = cc.rank_v;
    a.k_row = palu::latent_row_bytes(a.lat, a.r_k);
    a.v_row = palu::latent_row_bytes(a.lat, a.r_v);
    a.ks_row = palu::scale_row_bytes(a.lat, a.r_k);
    a.vs_row = palu::scale_row_bytes(a.lat, a.r_v);
    build_map(L, L.dset, c, zk_pool, zv_pool, zk_scales, zv_scales, a.gm);
    a.bk_box = a.r_k;
    for (int i = 0; i < a.gm.n; ++i)
      if (a.gm.rk[i] != a.r_k) a.bk_box = 64;   // mixed key ranks: boxes of 64 rows
    for (int j = 0; j < Q; j += a.qn) {
      a.qn = pass_queries(kind, Q - j);   // queries j .. j + qn - 1 of every sequence
      a.q = static_cast<const char*>(q) + (size_t)j * qrow * elt;
      a.q_pos = q_pos + j;
      a.out = static_cast<char*>(out) + (size_t)j * qrow * elt;
      a.lse = lse != nullptr ? lse + (size_t)j * a.H : nullptr;
      cudaError_t e = kind == 3   ? palu::launch_decode_fused(a, st)
                      : kind == 2 ? palu::launch_decode_tc(a, st)
                                  : palu::launch_decode_simt(a, st);
      if (e != cudaSuccess) return cuda_status(e);
      e = palu::launch_combine(a, st);
      if (e != cudaSuccess) return cuda_status(e);
    }
  }
  return PALU_OK;
}

}  // namespace

extern "C" {

const char* palu_status_string(palu_status s) {
  switch (s) {
    case PALU_OK: return "ok";
    case PALU_ERR_INVALID_ARG: return "invalid argument";
    case PALU_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case PALU_ERR_ALIGNMENT: return "pointer or row not 16-byte aligned";
    case PALU_ERR_WORKSPACE: return "workspace missing or too small";
    case PALU_ERR_CUDA: return "CUDA error";
    case PALU_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait timed out";
    case PALU_ERR_DEVICE_BOUNDS: return "a kernel found an index out of range";
  }
  return "unknown status";
}

const char* palu_last_cuda_error(void) { return g_cuda_err; }

int palu_decode_kernel_kind(const palu_config* cfg) { return kernel_kind(cfg); }

palu_status palu_debug_trace(void* buffer, size_t bytes, int tiles_per_cta) {
  if (buffer != nullptr && (tiles_per_cta <= 0 || bytes == 0)) return PALU_ERR_INVALID_ARG;
  palu::g_trace = palu::TraceSetting{buffer, buffer ? bytes : 0, buffer ? tiles_per_cta : 0};
  return PALU_OK;
}

uint64_t palu_kernel_launches(void) { return palu::g_launches.load(std::memory_order_relaxed); }

palu_status palu_debug_timeout_test(int64_t wait_cycles, int stall) {
  if (wait_cycles < 0) return PALU_ERR_INVALID_ARG;
  palu::g_timeout_test = palu::TimeoutTest{(long long)wait_cycles, stall != 0 ? 1 : 0};
  return PALU_OK;
}

palu_status palu_cache_strides(const palu_config* cfg, size_t* k_page_bytes, size_t* v_page_bytes,
                               size_t* k_scale_page_bytes, size_t* v_scale_page_bytes) {
  return palu_cache_strides_ranked(cfg, nullptr, nullptr, k_page_bytes, v_page_bytes, k_scale_page_bytes,
                                   v_scale_page_bytes, nullptr, nullptr);
}

palu_status palu_cache_strides_ranked(const palu_config* cfg, const int32_t* ranks_k, const int32_t* ranks_v,
                                      size_t* k_page_bytes, size_t* v_page_bytes, size_t* k_scale_page_bytes,
                                      size_t* v_scale_page_bytes, size_t* k_group_offsets,
                                      size_t* v_group_offsets) {
  Layer L;
  palu_status s = make_layer(cfg, ranks_k, ranks_v, &L);
  if (s != PALU_OK) return s;
  if (k_page_bytes) *k_page_bytes = (size_t)L.k_page;
  if (v_page_bytes) *v_page_bytes = (size_t)L.v_page;
  if (k_scale_page_bytes) *k_scale_page_bytes = (size_t)L.ks_page;
  if (v_scale_page_bytes) *v_scale_page_bytes = (size_t)L.vs_page;
  for (int g = 0; g < L.G; ++g) {
    if (k_group_offsets) k_group_offsets[g] = (size_t)L.k_off[g];
    if (v_group_offsets) v_group_offsets[g] = (size_t)L.v_off[g];
  }
  return PALU_OK;
}

palu_status palu_compress_workspace_size(const palu_config* cfg, int n_tokens, int d_model,
                                         size_t* bytes) {
  return palu_compress_ranked_workspace_size(cfg, nullptr, nullptr, n_tokens, d_model, bytes);
}

palu_status palu_compress_ranked_workspace_size(const palu_config* cfg, const int32_t* ranks_k,
                                                const int32_t* ranks_v, int n_tokens, int d_model, size_t* bytes) {
  Layer L;
  palu_status s = make_layer(cfg, ranks_k, ranks_v, &L);
  if (s != PALU_OK) return s;
  if (bytes == nullptr || n_tokens < 0 || d_model <= 0) return PALU_ERR_INVALID_ARG;
  *bytes = compress_workspace(L, n_tokens, d_model);
  return PALU_OK;
}

palu_status palu_compress_append(const palu_config* cfg, int n_tokens, int d_model, const void* x,
                                 const void* A_k, const void* A_v, const int32_t* slot_mapping,
                                 const int32_t* positions, void* zk_pool, void* zv_pool,
                                 void* zk_scales, void* zv_scales, int32_t* pos_pool, int num_pages,
                                 void* workspace, size_t workspace_bytes, palu_stream_t stream) {
  return palu_compress_append_ranked(cfg, nullptr, nullptr, n_tokens, d_model, x, A_k, A_v, slot_mapping, positions,
                                     zk_pool, zv_pool, zk_scales, zv_scales, pos_pool, num_pages, workspace,
                                     workspace_bytes, stream);
}

palu_status palu_compress_append_ranked(const palu_config* cfg, const int32_t* ranks_k, const int32_t* ranks_v,
                                        int n_tokens, int d_model, const void* x, const void* A_k, const void* A_v,
                                        const int32_t* slot_mapping, const int32_t* positions, void* zk_pool,
                                        void* zv_pool, void* zk_scales, void* zv_scales, int32_t* pos_pool,
                                        int num_pages, void* workspace, size_t workspace_bytes,
                                        palu_stream_t stream) {
  Layer L;
  palu_status s = make_layer(cfg, ranks_k, ranks_v, &L);
  if (s != PALU_OK) return s;
  return compress_layer(L, n_tokens, d_model, x, A_k, A_v, slot_mapping, positions, zk_pool, zv_pool, zk_scales,
                        zv_scales, pos_pool, num_pages, workspace, workspace_bytes, stream);
}

palu_status palu_decode_num_splits(const palu_config* cfg, int batch, int max_pages, int* num_splits) {
  palu_status s = check_config(cfg);
  if (s != PALU_OK) return s;
  if (num_splits == nullptr || batch < 0 || max_pages <= 0) return PALU_ERR_INVALID_ARG;
  *num_splits = auto_splits(cfg, batch, max_pages, kernel_kind(cfg));
  return PALU_OK;
}

palu_status palu_decode_workspace_size(const palu_config* cfg, int batch, int max_pages,
                                       int num_splits, size_t* bytes) {
  return palu_decode_ranked_workspace_size(cfg, nullptr, nullptr, batch, 1, max_pages, num_splits, bytes);
}

palu_status palu_decode_multi_workspace_size(const palu_config* cfg, int batch, int num_queries, int max_pages,
                                             int num_splits, size_t* bytes) {
  return palu_decode_ranked_workspace_size(cfg, nullptr, nullptr, batch, num_queries, max_pages, num_splits,
                                           bytes);
}

palu_status palu_decode_ranked_workspace_size(const palu_config* cfg, const int32_t* ranks_k,
                                              const int32_t* ranks_v, int batch, int num_queries, int max_pages,
                                              int num_splits, size_t* bytes) {
  Layer L;
  palu_status s = make_layer(cfg, ranks_k, ranks_v, &L);
  if (s != PALU_OK) return s;
  if (bytes == nullptr || batch < 0 || max_pages <= 0 || num_splits < 0 || num_queries < 1 ||
      num_queries > kMaxQueries)
    return PALU_ERR_INVALID_ARG;
  *bytes = decode_workspace(L, batch, num_queries, max_pages, num_splits, nullptr);
  return PALU_OK;
}

palu_status palu_decode_attn(const palu_config* cfg, int batch, const void* q, const int32_t* q_pos,
                             const void* zk_pool, const void* zv_pool, const void* zk_scales,
                             const void* zv_scales, const int32_t* pos_pool,
                             const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                             int num_pages, const void* B_k, const void* B_v, void* out, float* lse,
                             void* workspace, size_t workspace_bytes, int num_splits,
                             palu_stream_t stream) {
  return palu_decode_attn_ranked(cfg, nullptr, nullptr, batch, 1, q, q_pos, zk_pool, zv_pool, zk_scales, zv_scales,
                                 pos_pool, page_table, max_pages, seq_lens, num_pages, B_k, B_v, out, lse, workspace,
                                 workspace_bytes, num_splits, stream);
}

palu_status palu_decode_attn_multi(const palu_config* cfg, int batch, int num_queries, const void* q,
                                   const int32_t* q_pos, const void* zk_pool, const void* zv_pool,
                                   const void* zk_scales, const void* zv_scales, const int32_t* pos_pool,
                                   const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                                   int num_pages, const void* B_k, const void* B_v, void* out, float* lse,
                                   void* workspace, size_t workspace_bytes, int num_splits,
                                   palu_stream_t stream) {
  return palu_decode_attn_ranked(cfg, nullptr, nullptr, batch, num_queries, q, q_pos, zk_pool, zv_pool, zk_scales,
                                 zv_scales, pos_pool, page_table, max_pages, seq_lens, num_pages, B_k, B_v, out, lse,
                                 workspace, workspace_bytes, num_splits, stream);
}

palu_status palu_decode_attn_ranked(const palu_config* cfg, const int32_t* ranks_k, const int32_t* ranks_v,
                                    int batch, int num_queries, const void* q, const int32_t* q_pos,
                                    const void* zk_pool, const void* zv_pool, const void* zk_scales,
                                    const void* zv_scales, const int32_t* pos_pool, const int32_t* page_table,
                                    int max_pages, const int32_t* seq_lens, int num_pages, const void* B_k,
                                    const void* B_v, void* out, float* lse, void* workspace,
                                    size_t workspace_bytes, int num_splits, palu_stream_t stream) {
  Layer L;
  palu_status s = make_layer(cfg, ranks_k, ranks_v, &L);
  if (s != PALU_OK) return s;
  return decode_layer(L, batch, num_queries, q, q_pos, zk_pool, zv_pool, zk_scales, zv_scales, pos_pool,
                      page_table, max_pages, seq_lens, num_pages, B_k, B_v, out, lse, workspace, workspace_bytes,
                      num_splits, stream);
}

palu_status palu_get_device_status(void* workspace, palu_stream_t stream, int32_t* detail) {
  if (workspace == nullptr) return PALU_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  palu::DevStatus host{};
  cudaError_t e = cudaMemcpyAsync(&host, workspace, 8, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, 8, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_status(e);
  if (detail) *detail = host.detail;
  if (host.code == PALU_ERR_DEVICE_TIMEOUT) return PALU_ERR_DEVICE_TIMEOUT;
  if (host.code != 0) return PALU_ERR_DEVICE_BOUNDS;
  return PALU_OK;
}

}  // extern "C"
