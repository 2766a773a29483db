// MSA oracle: a plain, slow, float64 CPU statement of MiniMax Sparse Attention.
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
// execute this file: only the tests, the package's smoke() check and the
// bench's CPU-baseline leg use it.  It shares no code, header, table or helper
// with the CUDA library; the only thing both sides see is the seeded input
// generator, which holds none of the method's arithmetic.
//
// What it computes follows two pages on MSA:
//   [P4] "MiniMax M3 的 MSA 与阶跃 Step 3.7 Flash 的 MFA" (ai.air7.fun),
//        section "MSA：稀疏注意力的一种极简实现" (first layer = selection,
//        second layer = computation).
//   [P5] "MiniMax goes sparse" (atlascloud.ai), section 1
//        "圖表揭示的本質：兩階段處理，先選擇後計算", step 1 (index branch) and
//        step 2 (sparse branch).
// Every formula on those pages was lost when they were extracted from HTML;
// the readings taken where they are silent are listed beside each function.
//
// Conventions (all host memory, dense row-major, bf16 passed as raw uint16):
//   q      [batch, n_q, H, d]        k, v   [batch, max_kv, h, d]
//   q_idx  [batch, n_q, h, d_idx]    k_idx  [batch, max_kv, d_idx]
//   a "row" is one query position (b, t); its absolute position is
//   p = L_b - n_q + t, where L_b is the KV length of sequence b.
//   query head hq belongs to GQA group g = hq / (H / h) (contiguous groups:
//   [P5] step 2 and [P4] both say heads Q1..Q3 share I1 and Q4..Q6 share I2).
//
// Parity status: every function below is pinned by the CPU tests (closed
// forms, library routines, brute force and invariants); none is unpinned.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

struct Cfg {
  int batch, n_q, max_kv, H, h, d, d_idx, block, topk, causal, force_own;
  double scale;
};

// bf16 -> double: a bf16 value is the upper half of an IEEE binary32.
double bf(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

const double kNegInf = -std::numeric_limits<double>::infinity();

long kv_len(const Cfg& c, const int32_t* seq_lens, int b) {
  return seq_lens ? static_cast<long>(seq_lens[b]) : static_cast<long>(c.max_kv);
}

long nblk_max(const Cfg& c) { return (c.max_kv + c.block - 1) / c.block; }

// Number of blocks the query at absolute position p may look at.  Causal
// reading: a block is visible if its first token is at or before p; without
// the causal flag every block holding tokens < L_b is visible.
long frontier(const Cfg& c, long L, long p) {
  long nb = (L + c.block - 1) / c.block;
  if (!c.causal) return nb;
  if (p < 0) return 0;
  return std::min(nb, p / c.block + 1);
}

// Token j is a key the query at p may attend to.
bool key_visible(const Cfg& c, long L, long p, long j) {
  if (j < 0 || j >= L) return false;
  if (c.causal && j > p) return false;
  return true;
}

}  // namespace

extern "C" {

// Layout of the configuration struct shared with the Python wrapper.
typedef struct {
  int32_t batch, n_q, max_kv, H, h, d, d_idx, block, topk, causal, force_own;
  double scale;  // softmax scale; <= 0 means 1/sqrt(d)
} oracle_cfg_t;

static Cfg to_cfg(const oracle_cfg_t* o) {
  Cfg c{o->batch, o->n_q, o->max_kv, o->H, o->h, o->d, o->d_idx, o->block, o->topk,
        o->causal, o->force_own, o->scale};
  if (!(c.scale > 0.0)) c.scale = 1.0 / std::sqrt(static_cast<double>(c.d));
  return c;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// Stage 1a + 1b: index scores and Block Max Pool ([P4] first layer; [P5] step 1).
// For the row (b, t) and group g the token score is the plain inner product
// <q_idx[b,t,g,:], k_idx[b,j,:]>: one index query per GQA group against the
// single-head index key that all heads share.  No scale and no activation are
// applied (the formula is lost on the pages; a positive scale would not change
// the selection).  Block Max Pool takes, for block beta, the maximum token
// score over the tokens of that block the query may see (causal mask applied
// before pooling, so the query's own block pools only tokens j <= p).  Blocks
// with no visible token hold -inf.
// out: [nrows, h, nblk_max] doubles.
int oracle_block_scores(const oracle_cfg_t* oc, const int32_t* seq_lens, const uint16_t* q_idx,
                        const uint16_t* k_idx, int nrows, const int32_t* rows_b,
                        const int32_t* rows_t, double* out) {
  const Cfg c = to_cfg(oc);
  const long NB = nblk_max(c);
#pragma omp parallel for schedule(dynamic)
  for (long rg = 0; rg < static_cast<long>(nrows) * c.h; ++rg) {
    const int r = static_cast<int>(rg / c.h), g = static_cast<int>(rg % c.h);
    const int b = rows_b[r], t = rows_t[r];
    const long L = kv_len(c, seq_lens, b);
    const long p = L - c.n_q + t;
    const uint16_t* qv = q_idx + ((static_cast<long>(b) * c.n_q + t) * c.h + g) * c.d_idx;
    double* o = out + rg * NB;
    for (long beta = 0; beta < NB; ++beta) {
      double best = kNegInf;
      for (long j = beta * c.block; j < (beta + 1) * c.block; ++j) {
        if (!key_visible(c, L, p, j)) continue;
        const uint16_t* kv = k_idx + (static_cast<long>(b) * c.max_kv + j) * c.d_idx;
        double s = 0.0;
        for (int e = 0; e < c.d_idx; ++e) s += bf(qv[e]) * bf(kv[e]);
        best = std::max(best, s);
      }
      o[beta] = best;
    }
  }
  return 0;
}

// Stage 1c: TopK over block scores ([P4] first layer; [P5] step 1, "TopK
// decides which KV blocks this layer and this GQA group keep").
// Candidates are the blocks before the causal frontier F.  They are ordered by
// score, larger first, and among equal scores the lower block id first.  With
// force_own set, the query's own block floor(p / block) is placed first.  The
// first m = min(topk, F) candidates are taken and written in ascending block
// id order; the remaining topk - m slots hold -1.
// scores: [nrows, h, nblk_max]; ids: [nrows, h, topk].
int oracle_select(const oracle_cfg_t* oc, const int32_t* seq_lens, const double* scores,
                  int nrows, const int32_t* rows_b, const int32_t* rows_t, int32_t* ids) {
  const Cfg c = to_cfg(oc);
  const long NB = nblk_max(c);
#pragma omp parallel for schedule(dynamic)
  for (long rg = 0; rg < static_cast<long>(nrows) * c.h; ++rg) {
    const int r = static_cast<int>(rg / c.h);
    const int b = rows_b[r], t = rows_t[r];
    const long L = kv_len(c, seq_lens, b);
    const long p = L - c.n_q + t;
    const long F = frontier(c, L, p);
    const double* s = scores + rg * NB;
    std::vector<long> cand;
    for (long beta = 0; beta < F; ++beta) cand.push_back(beta);
    std::stable_sort(cand.begin(), cand.end(), [&](long x, long y) {
      if (s[x] != s[y]) return s[x] > s[y];
      return x < y;
    });
    if (c.force_own && F > 0) {
      const long own = p / c.block;
      auto it = std::find(cand.begin(), cand.end(), own);
      if (it != cand.end()) {
        cand.erase(it);
        cand.insert(cand.begin(), own);
      }
    }
    const long m = std::min<long>(c.topk, F);
    std::vector<long> pick(cand.begin(), cand.begin() + m);
    std::sort(pick.begin(), pick.end());
    int32_t* o = ids + rg * c.topk;
    for (long i = 0; i < c.topk; ++i) o[i] = i < m ? static_cast<int32_t>(pick[i]) : -1;
  }
  return 0;
}

// Softmax attention of one query head over an explicit key list, float64 with
// max subtraction.  Writes d outputs and the natural-log sum of exponentials.
static void attend(const Cfg& c, const uint16_t* qv, const uint16_t* k, const uint16_t* v, int b,
                   int g, const std::vector<long>& keys, double* o, double* lse) {
  for (int e = 0; e < c.d; ++e) o[e] = 0.0;
  if (keys.empty()) {
    *lse = kNegInf;
    return;
  }
  std::vector<double> z(keys.size());
  double zmax = kNegInf;
  for (size_t i = 0; i < keys.size(); ++i) {
    const uint16_t* kv = k + ((static_cast<long>(b) * c.max_kv + keys[i]) * c.h + g) * c.d;
    double s = 0.0;
    for (int e = 0; e < c.d; ++e) s += bf(qv[e]) * bf(kv[e]);
    z[i] = c.scale * s;
    zmax = std::max(zmax, z[i]);
  }
  double denom = 0.0;
  for (size_t i = 0; i < keys.size(); ++i) denom += std::exp(z[i] - zmax);
  for (size_t i = 0; i < keys.size(); ++i) {
    const double w = std::exp(z[i] - zmax) / denom;
    const uint16_t* vv = v + ((static_cast<long>(b) * c.max_kv + keys[i]) * c.h + g) * c.d;
    for (int e = 0; e < c.d; ++e) o[e] += w * bf(vv[e]);
  }
  *lse = zmax + std::log(denom);
}

// Stage 2: the sparse branch ([P4] second layer; [P5] step 2).  For query head
// hq of group g, the keys are the tokens of the blocks listed in
// ids[row, g, :] (entries < 0 are empty slots) that the query may see; the
// output is ordinary softmax attention with scale c.scale over the raw K/V of
// those tokens.  Every head of a group uses that group's one selection.
// ids: [nrows, h, topk]; out: [nrows, H, d]; lse: [nrows, H].
int oracle_sparse_attn(const oracle_cfg_t* oc, const int32_t* seq_lens, const uint16_t* q,
                       const uint16_t* k, const uint16_t* v, int nrows, const int32_t* rows_b,
                       const int32_t* rows_t, const int32_t* ids, double* out, double* lse) {
  const Cfg c = to_cfg(oc);
  const int G = c.H / c.h;
#pragma omp parallel for schedule(dynamic)
  for (long rh = 0; rh < static_cast<long>(nrows) * c.H; ++rh) {
    const int r = static_cast<int>(rh / c.H), hq = static_cast<int>(rh % c.H);
    const int g = hq / G;
    const int b = rows_b[r], t = rows_t[r];
    const long L = kv_len(c, seq_lens, b);
    const long p = L - c.n_q + t;
    const int32_t* sel = ids + (static_cast<long>(r) * c.h + g) * c.topk;
    std::vector<long> blocks;
    for (int i = 0; i < c.topk; ++i)
      if (sel[i] >= 0) blocks.push_back(sel[i]);
    std::sort(blocks.begin(), blocks.end());
    blocks.erase(std::unique(blocks.begin(), blocks.end()), blocks.end());
    std::vector<long> keys;
    for (long beta : blocks)
      for (long j = beta * c.block; j < (beta + 1) * c.block; ++j)
        if (key_visible(c, L, p, j)) keys.push_back(j);
    const uint16_t* qv = q + ((static_cast<long>(b) * c.n_q + t) * c.H + hq) * c.d;
    attend(c, qv, k, v, b, g, keys, out + rh * c.d, lse + rh);
  }
  return 0;
}

// Textbook dense GQA softmax attention (causal when c.causal), written out
// separately from the sparse branch: every visible token is a key.
int oracle_dense_attn(const oracle_cfg_t* oc, const int32_t* seq_lens, const uint16_t* q,
                      const uint16_t* k, const uint16_t* v, int nrows, const int32_t* rows_b,
                      const int32_t* rows_t, double* out, double* lse) {
  const Cfg c = to_cfg(oc);
  const int G = c.H / c.h;
#pragma omp parallel for schedule(dynamic)
  for (long rh = 0; rh < static_cast<long>(nrows) * c.H; ++rh) {
    const int r = static_cast<int>(rh / c.H), hq = static_cast<int>(rh % c.H);
    const int b = rows_b[r], t = rows_t[r];
    const long L = kv_len(c, seq_lens, b);
    const long p = L - c.n_q + t;
    std::vector<long> keys;
    for (long j = 0; j < L; ++j)
      if (key_visible(c, L, p, j)) keys.push_back(j);
    const uint16_t* qv = q + ((static_cast<long>(b) * c.n_q + t) * c.H + hq) * c.d;
    attend(c, qv, k, v, b, hq / G, keys, out + rh * c.d, lse + rh);
  }
  return 0;
}

// The whole method for a list of rows: block scores, selection, then the
// sparse branch on that selection (used by the CPU baseline timing).
int oracle_forward(const oracle_cfg_t* oc, const int32_t* seq_lens, const uint16_t* q,
                   const uint16_t* k, const uint16_t* v, const uint16_t* q_idx,
                   const uint16_t* k_idx, int nrows, const int32_t* rows_b, const int32_t* rows_t,
                   int32_t* ids, double* out, double* lse) {
  const Cfg c = to_cfg(oc);
  std::vector<double> scores(static_cast<size_t>(nrows) * c.h * nblk_max(c));
  oracle_block_scores(oc, seq_lens, q_idx, k_idx, nrows, rows_b, rows_t, scores.data());
  oracle_select(oc, seq_lens, scores.data(), nrows, rows_b, rows_t, ids);
  return oracle_sparse_attn(oc, seq_lens, q, k, v, nrows, rows_b, rows_t, ids, out, lse);
}

}  // extern "C"
