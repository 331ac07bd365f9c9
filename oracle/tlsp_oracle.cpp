// fp64 CPU oracle for the MC-Sparse attention hot path.
//
// TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls
// this file: only the tests, the package's smoke check and the benchmark's CPU
// baseline leg do. It shares no code, header or table with the CUDA library.
//
// Everything is double precision, one (batch, head) slice per call, row-major
// with the head dimension contiguous. Each function is the plain definition of
// one step of the method as the MC-Sparse review ("Deconstructing and Closing
// the Dense-Sparse Attention Gap in Diffusion Transformers", section 3,
// "Method & Key Results") states it; where the page leaves a step open the
// reading taken is written beside it.
//
// Pins (checks against something other than this file) live in
// tests/test_oracle_pins.py. Parity unpinned: none of the functions below;
// the "similarity-maximising" quality claim of the grouping has no number on
// the page and is only reported.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <numeric>
#include <vector>

namespace {

double dot(const double* a, const double* b, int64_t d) {
  double s = 0.0;
  for (int64_t c = 0; c < d; ++c) s += a[c] * b[c];
  return s;
}

// Leading principal direction of the rows X[members] by power iteration.
// Reading (page silent on "Fast" PDDP): start from the normalised ones vector,
// run a fixed n_iter iterations of w = C^T (C v), v = w / |w| with C the
// centred rows; if |w| <= 1e-30 * n the node has no spread and v = e_0.
// The sign is fixed so that the component of largest magnitude (lowest
// channel on ties) is positive.
void principal_direction(const double* X, int64_t d, const std::vector<int32_t>& members,
                         int n_iter, std::vector<double>& mu, std::vector<double>& v) {
  const int64_t n = (int64_t)members.size();
  mu.assign(d, 0.0);
  for (int32_t i : members)
    for (int64_t c = 0; c < d; ++c) mu[c] += X[(int64_t)i * d + c];
  for (int64_t c = 0; c < d; ++c) mu[c] /= (double)n;

  v.assign(d, 1.0 / std::sqrt((double)d));
  std::vector<double> w(d), xc(d);
  for (int it = 0; it < n_iter; ++it) {
    std::fill(w.begin(), w.end(), 0.0);
    for (int32_t i : members) {
      const double* x = X + (int64_t)i * d;
      for (int64_t c = 0; c < d; ++c) xc[c] = x[c] - mu[c];
      const double u = dot(xc.data(), v.data(), d);          // (C v)_i
      for (int64_t c = 0; c < d; ++c) w[c] += u * xc[c];      // C^T (C v)
    }
    const double nw = std::sqrt(dot(w.data(), w.data(), d));
    if (nw <= 1e-30 * (double)n) {
      std::fill(v.begin(), v.end(), 0.0);
      v[0] = 1.0;
      break;
    }
    for (int64_t c = 0; c < d; ++c) v[c] = w[c] / nw;
  }
  int64_t cmax = 0;
  for (int64_t c = 1; c < d; ++c)
    if (std::fabs(v[c]) > std::fabs(v[cmax])) cmax = c;
  if (v[cmax] < 0)
    for (int64_t c = 0; c < d; ++c) v[c] = -v[c];
}

struct Node {
  std::vector<int32_t> tokens;  // ascending token ids
  int64_t slots;                // number of leaf groups this node will hold
};

// Reading of "equal-size, tile-aligned groups" for N not divisible by the
// group size: a node with s slots sends its floor(s/2) * gs lowest-ranked
// tokens left (floor(s/2) slots) and the rest right (ceil(s/2) slots), so
// every group is full except the rightmost one.
void split_node(const Node& node, int64_t gs, const std::vector<double>& p, Node& left,
                Node& right) {
  std::vector<int32_t> order = node.tokens;
  std::sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
    const double pa = p[a], pb = p[b];
    if (pa != pb) return pa < pb;  // -0 == +0 here: ties fall to the index
    return a < b;
  });
  const int64_t left_slots = node.slots / 2;
  const int64_t n_left = left_slots * gs;
  left.tokens.assign(order.begin(), order.begin() + n_left);
  right.tokens.assign(order.begin() + n_left, order.end());
  std::sort(left.tokens.begin(), left.tokens.end());
  std::sort(right.tokens.begin(), right.tokens.end());
  left.slots = left_slots;
  right.slots = node.slots - left_slots;
}

// Shared driver of grouping and of its replay: `project` fills p[token] for
// the tokens of a node split at `level`.
template <class Project>
int64_t run_pddp(int64_t n, int64_t gs, Project project, int32_t* groups) {
  const int64_t G = (n + gs - 1) / gs;
  std::vector<Node> level_nodes(1);
  level_nodes[0].tokens.resize(n);
  std::iota(level_nodes[0].tokens.begin(), level_nodes[0].tokens.end(), 0);
  level_nodes[0].slots = G;
  std::vector<double> p(n, 0.0);
  int64_t level = 0;
  for (;;) {
    bool any_split = false;
    for (const Node& nd : level_nodes) any_split |= nd.slots > 1;
    if (!any_split) break;
    std::vector<Node> next;
    for (const Node& nd : level_nodes) {
      if (nd.slots == 1) {
        next.push_back(nd);
        continue;
      }
      project(level, nd.tokens, p);
      Node l, r;
      split_node(nd, gs, p, l, r);
      next.push_back(std::move(l));
      next.push_back(std::move(r));
    }
    level_nodes.swap(next);
    ++level;
  }
  // Leaves left to right; the ragged rightmost leaf is padded with -1.
  int64_t pos = 0;
  for (const Node& nd : level_nodes) {
    for (int64_t r = 0; r < gs; ++r)
      groups[pos + r] = r < (int64_t)nd.tokens.size() ? nd.tokens[r] : -1;
    pos += gs;
  }
  return level;
}

}  // namespace

extern "C" {

// Dense softmax attention (the anchor step's "dense attention output").
// For each query row r: s_j = (q_r . k_j) / sqrt(d) over all nkv keys (reading:
// the usual 1/sqrt(d) scale, bidirectional, no mask), O_r = sum_j softmax(s)_j v_j
// and LSE_r = log sum_j exp(s_j).
void orc_dense_rows(int64_t nrows, int64_t nkv, int64_t d, const double* Q, const double* K,
                    const double* V, double* O, double* LSE) {
  const double scale = 1.0 / std::sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < nrows; ++r) {
    std::vector<double> s(nkv);
    const double* q = Q + r * d;
    double m = -INFINITY;
    for (int64_t j = 0; j < nkv; ++j) {
      s[j] = dot(q, K + j * d, d) * scale;
      m = std::max(m, s[j]);
    }
    double l = 0.0;
    for (int64_t j = 0; j < nkv; ++j) {
      s[j] = std::exp(s[j] - m);
      l += s[j];
    }
    double* o = O + r * d;
    std::fill(o, o + d, 0.0);
    for (int64_t j = 0; j < nkv; ++j) {
      const double pj = s[j] / l;
      const double* vj = V + j * d;
      for (int64_t c = 0; c < d; ++c) o[c] += pj * vj[c];
    }
    LSE[r] = m + std::log(l);
  }
}

// Exact KV score of one query group (reading of the page's "exact attention
// score" used for selection instead of mean pooling): the summed softmax
// probability the group's queries put on each key,
// S[j] = sum_r exp((q_r . k_j) / sqrt(d) - LSE_r).
void orc_group_scores(int64_t nrows, int64_t nkv, int64_t d, const double* Qg, const double* LSEg,
                      const double* K, double* S) {
  const double scale = 1.0 / std::sqrt((double)d);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < nkv; ++j) {
    double acc = 0.0;
    for (int64_t r = 0; r < nrows; ++r) acc += std::exp(dot(Qg + r * d, K + j * d, d) * scale - LSEg[r]);
    S[j] = acc;
  }
}

// Token-level KV selection: the k keys of largest score; equal scores go to
// the lower key index (reading: fixed tie order). The chosen set is returned
// in ascending key order (reading: the selection is a set).
void orc_topk(int64_t n, const double* s, int64_t k, int32_t* idx) {
  std::vector<int32_t> order(n);
  std::iota(order.begin(), order.end(), 0);
  std::sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
    if (s[a] != s[b]) return s[a] > s[b];
    return a < b;
  });
  const int64_t kk = std::min(k, n);
  std::sort(order.begin(), order.begin() + kk);
  for (int64_t t = 0; t < kk; ++t) idx[t] = order[t];
}

// Sparse attention of query rows over the selected keys only; the softmax is
// renormalised over the selection (reading of "discarded tail": the keys left
// out contribute nothing), so selecting every key gives dense attention.
void orc_sparse_rows(int64_t nrows, int64_t d, const double* Q, const double* K, const double* V,
                     int64_t nsel, const int32_t* idx, double* O) {
  const double scale = 1.0 / std::sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < nrows; ++r) {
    std::vector<double> s(nsel);
    const double* q = Q + r * d;
    double m = -INFINITY;
    for (int64_t t = 0; t < nsel; ++t) {
      s[t] = dot(q, K + (int64_t)idx[t] * d, d) * scale;
      m = std::max(m, s[t]);
    }
    double l = 0.0;
    for (int64_t t = 0; t < nsel; ++t) {
      s[t] = std::exp(s[t] - m);
      l += s[t];
    }
    double* o = O + r * d;
    std::fill(o, o + d, 0.0);
    for (int64_t t = 0; t < nsel; ++t) {
      const double pt = s[t] / l;
      const double* vt = V + (int64_t)idx[t] * d;
      for (int64_t c = 0; c < d; ++c) o[c] += pt * vt[c];
    }
  }
}

// Centre and leading principal direction of the rows X[members[0..m)].
void orc_pddp_direction(int64_t m, const int32_t* members, int64_t d, const double* X, int n_iter,
                        double* mu_out, double* v_out) {
  std::vector<int32_t> mem(members, members + m);
  std::vector<double> mu, v;
  principal_direction(X, d, mem, n_iter, mu, v);
  std::copy(mu.begin(), mu.end(), mu_out);
  std::copy(v.begin(), v.end(), v_out);
}

// Tile-aligned query grouping by principal direction divisive partitioning
// of one head's queries X [n, d] into G = ceil(n / gs) groups. Each node is
// centred, projected on its leading principal direction and cut by rank (ties
// by token index) so that the left child holds floor(s/2) full groups.
// groups [G * gs]: leaves left to right, tokens ascending inside a leaf, -1
// pads the ragged last leaf. trace (optional) [max_levels * n] receives the
// projection of every token of a node split at each level (0 elsewhere).
// Returns the number of levels.
int64_t orc_pddp(int64_t n, int64_t d, const double* X, int64_t gs, int n_iter, int32_t* groups,
                 double* trace, int64_t max_levels) {
  if (trace) std::fill(trace, trace + max_levels * n, 0.0);
  auto project = [&](int64_t level, const std::vector<int32_t>& toks, std::vector<double>& p) {
    std::vector<double> mu, v;
    principal_direction(X, d, toks, n_iter, mu, v);
    std::vector<double> xc(d);
    for (int32_t i : toks) {
      for (int64_t c = 0; c < d; ++c) xc[c] = X[(int64_t)i * d + c] - mu[c];
      p[i] = dot(xc.data(), v.data(), d);
      if (trace && level < max_levels) trace[level * n + i] = p[i];
    }
  };
  return run_pddp(n, gs, project, groups);
}

// The same recursion, but each node is cut on projections supplied by the
// caller (proj [levels * n], fp32 as produced by another implementation)
// instead of computing them. If X is given, own [levels * n] receives this
// oracle's fp64 projections for the very same nodes (0 elsewhere).
int64_t orc_pddp_replay(int64_t n, int64_t gs, int64_t levels, const float* proj, int32_t* groups,
                        int64_t d, const double* X, int n_iter, double* own) {
  if (own) std::fill(own, own + levels * n, 0.0);
  auto project = [&](int64_t level, const std::vector<int32_t>& toks, std::vector<double>& p) {
    for (int32_t i : toks) p[i] = level < levels ? (double)proj[level * n + i] : 0.0;
    if (X && own && level < levels) {
      std::vector<double> mu, v, xc(d);
      principal_direction(X, d, toks, n_iter, mu, v);
      for (int32_t i : toks) {
        for (int64_t c = 0; c < d; ++c) xc[c] = X[(int64_t)i * d + c] - mu[c];
        own[level * n + i] = dot(xc.data(), v.data(), d);
      }
    }
  };
  return run_pddp(n, gs, project, groups);
}

}  // extern "C"
