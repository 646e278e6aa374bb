// plan.inl -- host planner: tiling of the token grid, tile <-> token index maps,
// blend weights w-bar, and the per-row tables the kernels read (attention row map,
// RoPE coordinates).  Included by tileshare.cu.
//
// [TileShare] abstract: a fixed-window decoder runs at deployment resolution as
// overlapping tiles, and the tokens of overlap bands are blended with the released
// weights; Fig. 2: an overlap token is stored once and attended in every window
// covering it.  Readings (the pages print neither rule):
//   placement  per axis n = ceil((G - w) / s) + 1 tiles (1 if w == G) at origins
//              min(i*s, G - w), the last tile flush with the far edge;
//   weights    separable linear ramps: along an axis, a tile overlapped by its
//              previous neighbour over o_p tokens and by its next one over o_n
//              tokens weighs local position p by (p + 1) / (o_p + 1) for p < o_p
//              and by (w - p) / (o_n + 1) for p >= w - o_n (product where both
//              apply), 1 elsewhere; the tile weight is the product over axes,
//              normalised to sum 1 over the tiles covering the token.
//   registers  each tile has R register tokens ([TileShare] Tab. S1: one set per
//              tile); the per-tile state is [R registers | Nw window slots] and the
//              shared state [U grid tokens | T*R registers, tile t's at U + t*R].
// Weights are computed in double and stored as float.
#pragma once

#include <cmath>
#include <cstring>
#include <vector>

struct ts_plan_s {
  int grid[3], win[3], stride[3];
  int T, U, Nw, N, nnz, max_cover, device;
  int R = 1;                     // register tokens per tile; N = Nw + R
  int G = 0;                     // register rows of the shared state, T * R
  int run;                       // slots 1 + k*run .. are runs of consecutive shared rows (0: none)
  int rule;                      // blend rule: 0 linear ramp (normalised), 1 hard stitching (one tile per token)
  std::vector<int> origins, tile_tok, slot_pos, tok_ptr, tok_ent;
  std::vector<float> wbar;
  std::vector<int> rowmap;       // [T*N] shared-layout row of slot s of tile t (s < R: U + t*R + s)
  std::vector<int> pos_shared;   // [(U+G)*4] RoPE coordinates of shared rows
  std::vector<int> pos_tiled;    // [(T*N)*4] RoPE coordinates of per-tile rows
  // device copies (on `device`)
  int* d_tok_ptr = nullptr;
  int* d_tok_ent = nullptr;
  float* d_wbar = nullptr;
  int* d_rowmap = nullptr;
  int* d_pos_shared = nullptr;
  int* d_pos_tiled = nullptr;
};

namespace tsplan {

inline std::vector<int> axis_origins(int G, int w, int s) {
  std::vector<int> o;
  if (w == G) {
    o.push_back(0);
    return o;
  }
  const int n = (G - w + s - 1) / s + 1;
  for (int i = 0; i < n; ++i) o.push_back(std::min(i * s, G - w));
  return o;
}

// unnormalised weight of tile i at local position p along one axis
inline std::vector<double> axis_weights(const std::vector<int>& o, int w) {
  const int n = static_cast<int>(o.size());
  std::vector<double> r(static_cast<size_t>(n) * w, 1.0);
  for (int i = 0; i < n; ++i) {
    const int op = i > 0 ? std::max(o[i - 1] + w - o[i], 0) : 0;
    const int on = i + 1 < n ? std::max(o[i] + w - o[i + 1], 0) : 0;
    for (int p = 0; p < w; ++p) {
      double v = 1.0;
      if (p < op) v *= static_cast<double>(p + 1) / static_cast<double>(op + 1);
      if (p >= w - on) v *= static_cast<double>(w - p) / static_cast<double>(on + 1);
      r[static_cast<size_t>(i) * w + p] = v;
    }
  }
  return r;
}

// Fill the host side of a plan; returns false on an uncovered token.
inline bool build(ts_plan_s& P) {
  const int F = P.grid[0], H = P.grid[1], W = P.grid[2];
  const int wf = P.win[0], wh = P.win[1], ww = P.win[2];
  const std::vector<int> of = axis_origins(F, wf, P.stride[0]);
  const std::vector<int> oh = axis_origins(H, wh, P.stride[1]);
  const std::vector<int> ow = axis_origins(W, ww, P.stride[2]);
  const std::vector<double> rf = axis_weights(of, wf), rh = axis_weights(oh, wh), rw = axis_weights(ow, ww);
  const int nf = static_cast<int>(of.size()), nh = static_cast<int>(oh.size()), nw = static_cast<int>(ow.size());
  P.T = nf * nh * nw;
  P.Nw = wf * wh * ww;
  P.N = P.Nw + P.R;
  P.G = P.T * P.R;
  P.U = F * H * W;
  P.nnz = P.T * P.Nw;
  P.slot_pos.assign(static_cast<size_t>(P.Nw) * 3, 0);
  for (int lf = 0, j = 0; lf < wf; ++lf)
    for (int ly = 0; ly < wh; ++ly)
      for (int lx = 0; lx < ww; ++lx, ++j) {
        P.slot_pos[3 * j] = lf;
        P.slot_pos[3 * j + 1] = ly;
        P.slot_pos[3 * j + 2] = lx;
      }
  P.origins.assign(static_cast<size_t>(P.T) * 3, 0);
  P.tile_tok.assign(static_cast<size_t>(P.T) * P.Nw, 0);
  std::vector<double> wraw(static_cast<size_t>(P.T) * P.Nw);
  for (int a = 0, t = 0; a < nf; ++a)
    for (int b = 0; b < nh; ++b)
      for (int c = 0; c < nw; ++c, ++t) {
        P.origins[3 * t] = of[a];
        P.origins[3 * t + 1] = oh[b];
        P.origins[3 * t + 2] = ow[c];
        for (int j = 0; j < P.Nw; ++j) {
          const int lf = P.slot_pos[3 * j], ly = P.slot_pos[3 * j + 1], lx = P.slot_pos[3 * j + 2];
          const size_t e = static_cast<size_t>(t) * P.Nw + j;
          P.tile_tok[e] = ((of[a] + lf) * H + (oh[b] + ly)) * W + (ow[c] + lx);
          wraw[e] = rf[static_cast<size_t>(a) * wf + lf] * rh[static_cast<size_t>(b) * wh + ly] *
                    rw[static_cast<size_t>(c) * ww + lx];
        }
      }
  // per-token totals and coverage, tiles in ascending order
  std::vector<double> total(P.U, 0.0);
  std::vector<int> cover(P.U, 0);
  for (size_t e = 0; e < wraw.size(); ++e) {
    total[P.tile_tok[e]] += wraw[e];
    cover[P.tile_tok[e]] += 1;
  }
  P.max_cover = 0;
  for (int u = 0; u < P.U; ++u) {
    if (cover[u] == 0) return false;
    P.max_cover = std::max(P.max_cover, cover[u]);
  }
  // hard stitching: the covering tile with the largest raw weight (first, i.e.
  // lowest, tile on ties) is the token's only entry, with weight 1
  std::vector<int> best_t;
  if (P.rule == 1) {
    best_t.assign(P.U, -1);
    std::vector<double> best_w(P.U, -1.0);
    for (int t = 0; t < P.T; ++t)
      for (int j = 0; j < P.Nw; ++j) {
        const size_t e = static_cast<size_t>(t) * P.Nw + j;
        const int u = P.tile_tok[e];
        if (wraw[e] > best_w[u]) {
          best_w[u] = wraw[e];
          best_t[u] = t;
        }
      }
    P.nnz = P.U;
  }
  // CSR over grid tokens; entries in ascending tile order
  P.tok_ptr.assign(P.U + 1, 0);
  for (int u = 0; u < P.U; ++u) P.tok_ptr[u + 1] = P.tok_ptr[u] + (P.rule == 1 ? 1 : cover[u]);
  P.tok_ent.assign(P.nnz, 0);
  P.wbar.assign(P.nnz, 0.f);
  std::vector<int> fill(P.tok_ptr.begin(), P.tok_ptr.end() - 1);
  for (int t = 0; t < P.T; ++t)
    for (int j = 0; j < P.Nw; ++j) {
      const size_t e = static_cast<size_t>(t) * P.Nw + j;
      const int u = P.tile_tok[e];
      if (P.rule == 1 && best_t[u] != t) continue;
      const int k = fill[u]++;
      P.tok_ent[k] = t * P.N + P.R + j;
      P.wbar[k] = P.rule == 1 ? 1.0f : static_cast<float>(wraw[e] / total[u]);
    }
  // attention row map of the shared layout and RoPE coordinates
  P.rowmap.assign(static_cast<size_t>(P.T) * P.N, 0);
  P.pos_tiled.assign(static_cast<size_t>(P.T) * P.N * 4, 0);
  for (int t = 0; t < P.T; ++t) {
    for (int i = 0; i < P.R; ++i) P.rowmap[static_cast<size_t>(t) * P.N + i] = P.U + t * P.R + i;
    for (int j = 0; j < P.Nw; ++j) {
      const size_t r = static_cast<size_t>(t) * P.N + P.R + j;
      P.rowmap[r] = P.tile_tok[static_cast<size_t>(t) * P.Nw + j];
      for (int a = 0; a < 3; ++a) P.pos_tiled[4 * r + a] = P.slot_pos[3 * j + a];
    }
  }
  // longest run length (64, 32, 16 or 8) such that every aligned group of slots
  // 1 + k*run, ..., run + k*run of every tile maps to consecutive shared rows
  P.run = 0;
  for (int L = 64; L >= 8 && !P.run; L >>= 1) {
    bool ok = true;
    for (int t = 0; t < P.T && ok; ++t)
      for (int j = 1; j < P.N - 1 && ok; ++j)
        if (j % L) ok = P.rowmap[static_cast<size_t>(t) * P.N + 1 + j] == P.rowmap[static_cast<size_t>(t) * P.N + j] + 1;
    if (ok) P.run = L;
  }
  P.pos_shared.assign(static_cast<size_t>(P.U + P.G) * 4, 0);
  for (int f = 0, u = 0; f < F; ++f)
    for (int y = 0; y < H; ++y)
      for (int x = 0; x < W; ++x, ++u) {
        P.pos_shared[4 * u] = f;
        P.pos_shared[4 * u + 1] = y;
        P.pos_shared[4 * u + 2] = x;
      }
  for (int t = 0; t < P.T; ++t)
    for (int i = 0; i < P.R; ++i)
      for (int a = 0; a < 3; ++a)
        P.pos_shared[4 * (static_cast<size_t>(P.U) + t * P.R + i) + a] = P.origins[3 * t + a];
  return true;
}

}  // namespace tsplan
