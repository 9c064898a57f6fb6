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

}  // namespace attn
