// Launch order of the attention kernels' (problem, tile) grids.
//
// A grid of P problems (batch x head, or sequence x head) by T tiles is
// launched as one dimension of P*T CTAs.  CTA number c walks groups of G
// problems; inside a group the tile index is the slow one and the problem the
// fast one:
//
//   group g = c / (G*T), r = c - g*G*T, size = min(G, P - g*G),
//   tile = r / size, problem = g*G + r % size.
//
// The CTAs resident at one time then belong to about G problems.  Every CTA
// of a problem streams the same operands (the forward's K and V, the
// backward's Q, dO and dQ accumulator), so G is chosen on the host so that G
// problems' streamed operands stay in L2.  G = P gives problem-fastest order
// over the whole grid.  Inside a group the tile order is kept, so causal
// grids still launch their heaviest tiles first.
//
// This header is plain C++ (no CUDA types) so that host code and host tests
// can use it as well as the kernels.
#pragma once

#ifdef __CUDACC__
#define ATTN_HD __host__ __device__ __forceinline__
#else
#define ATTN_HD inline
#endif

namespace attn {

// Bytes of L2 the streamed operands of one group may take: a quarter of the
// 126 MB L2, leaving room for the CTAs' own tiles and the write streams.
constexpr double kOrderL2Budget = 32.0 * 1024.0 * 1024.0;

// Maps linear CTA number c (c < problems * tiles <= 2^31 - 1) to its
// (problem, tile).  group is in [1, problems].
ATTN_HD void grouped_order(unsigned c, int problems, int tiles, int group, int* problem, int* tile) {
  const unsigned span = static_cast<unsigned>(group) * static_cast<unsigned>(tiles);
  const unsigned g = c / span;
  const unsigned r = c - g * span;
  const int first = static_cast<int>(g) * group;
  const int size = problems - first < group ? problems - first : group;
  *tile = static_cast<int>(r / static_cast<unsigned>(size));
  *problem = first + static_cast<int>(r % static_cast<unsigned>(size));
}

// Group size for problems that each stream bytes_per_problem from HBM: as
// many problems as fit the budget, at least one and at most all.
inline int order_group(double bytes_per_problem, int problems) {
  if (problems <= 1) return 1;
  if (!(bytes_per_problem > 0.0)) return problems;
  const double g = kOrderL2Budget / bytes_per_problem;
  if (g >= static_cast<double>(problems)) return problems;
  return g < 1.0 ? 1 : static_cast<int>(g);
}

// Persistent grids: `grid` CTAs share the units (problem, tile) of the
// launch order above.  The units are dealt in rounds of `grid` items; in
// round r CTA c takes item r * grid + c for even r and r * grid + grid-1-c
// for odd r (a snake: the CTA that took the last item of one round takes the
// first of the next).  Without folding an item is one unit, in launch order.
// With folding (causal grids, whose tiles get lighter along the order inside
// a group), item k of a group of S units is the pair of units k and S-1-k of
// that group: a heavy tile and a light one, so that every item carries about
// the same work and the CTAs' totals stay within about one item of each
// other.  Every unit belongs to exactly one item.
struct UnitPlan {
  int units;      // problems * tiles
  int span;       // units of a full group
  int per_group;  // items of a full group
  int items;
  int fold;
};

ATTN_HD UnitPlan unit_plan(int problems, int tiles, int group, int fold) {
  UnitPlan p;
  p.units = problems * tiles;
  p.span = group * tiles;
  p.fold = fold;
  p.per_group = fold ? (p.span + 1) / 2 : p.span;
  const int full = p.span > 0 ? p.units / p.span : 0;
  const int tail = p.units - full * p.span;
  p.items = full * p.per_group + (fold ? (tail + 1) / 2 : tail);
  return p;
}

// Unit slots each CTA walks (some of them empty).
ATTN_HD int unit_slots(const UnitPlan& p, unsigned grid) {
  const int rounds = static_cast<int>((static_cast<unsigned>(p.items) + grid - 1u) / grid);
  return p.fold ? 2 * rounds : rounds;
}

// Unit of slot s of CTA cta, or -1 for an empty slot.
ATTN_HD int unit_at(const UnitPlan& p, unsigned grid, unsigned cta, int s) {
  const int r = p.fold ? s >> 1 : s;
  const unsigned c = (r & 1) ? grid - 1u - cta : cta;
  const unsigned it = static_cast<unsigned>(r) * grid + c;  // unsigned: may pass 2^31 - 1
  if (it >= static_cast<unsigned>(p.items)) return -1;
  if (!p.fold) return static_cast<int>(it);
  const int g = static_cast<int>(it) / p.per_group;
  const int k = static_cast<int>(it) - g * p.per_group;
  const int g0 = g * p.span;
  const int size = p.units - g0 < p.span ? p.units - g0 : p.span;
  if ((s & 1) == 0) return g0 + k;
  return size - 1 - k != k ? g0 + size - 1 - k : -1;
}

}  // namespace attn
