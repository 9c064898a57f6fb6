"""The grouped launch order of the kernels' (problem, tile) grids
(exact_attention_150_b200/csrc/tile_order.h), compiled as plain C++ on the
host: every CTA number maps to a distinct (problem, tile), groups hold at most
G problems, the tile order inside a group is kept, and the group size follows
the L2 budget."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_attention_150_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <vector>
#include "tile_order.h"

#define EXPECT(cond) do { if (!(cond)) { std::printf("FAILED line %d: %s (P=%d T=%d G=%d)\n", __LINE__, #cond, P, T, G); return 1; } } while (0)

int check(int P, int T, int G) {
  std::vector<int> seen(static_cast<size_t>(P) * T, 0);
  int prev_group = -1, prev_tile = -1;
  for (unsigned c = 0; c < static_cast<unsigned>(P) * T; ++c) {
    int p = -1, t = -1;
    attn::grouped_order(c, P, T, G, &p, &t);
    EXPECT(p >= 0 && p < P && t >= 0 && t < T);
    EXPECT(seen[static_cast<size_t>(p) * T + t]++ == 0);
    const int g = p / G;
    EXPECT(g >= prev_group);                        // groups are walked in order
    if (g != prev_group) prev_tile = -1;
    EXPECT(t >= prev_tile);                         // tile order kept inside a group
    prev_group = g;
    prev_tile = t;
    if (G == P) EXPECT(p == static_cast<int>(c % P) && t == static_cast<int>(c / P));  // problem-fastest
  }
  return 0;
}

int main() {
  const int shapes[][2] = {{1, 1}, {1, 7}, {2, 1}, {3, 5}, {16, 128}, {128, 64}, {37, 11}, {64, 3}, {5, 128}};
  for (const auto& s : shapes) {
    const int P = s[0], T = s[1];
    for (int G = 1; G <= P; ++G)
      if (check(P, T, G)) return 1;
  }
  // Group sizes: the budget over the bytes per problem, in [1, problems].
  const double mb = 1024.0 * 1024.0;
  int P = 0, T = 0, G = 0;
  EXPECT(attn::order_group(4 * mb, 128) == 8);        // 16 heads x 8192 keys x d 128: K and V, 4 MB each problem
  EXPECT(attn::order_group(8 * mb, 16) == 4);
  EXPECT(attn::order_group(16.9 * mb, 16) == 1);
  EXPECT(attn::order_group(100 * mb, 16) == 1);       // larger than the budget: one problem at a time
  EXPECT(attn::order_group(1 * mb, 16) == 16);        // all fit: problem-fastest over the whole grid
  EXPECT(attn::order_group(0.0, 16) == 16);
  EXPECT(attn::order_group(4 * mb, 1) == 1);
  EXPECT(attn::order_group(4 * mb, 0) == 1);
  std::printf("ok\n");
  return 0;
}
"""


def test_grouped_order_is_a_bijection_in_tile_order(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no C++ compiler")
    src = tmp_path / "order.cpp"
    src.write_text(PROGRAM)
    exe = tmp_path / "order"
    subprocess.run([cxx, "-std=c++17", "-O1", "-Wall", "-Wextra", "-Werror", "-I", CSRC, str(src), "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr


PLAN_PROGRAM = r"""
#include <algorithm>
#include <cstdio>
#include <vector>
#include "tile_order.h"

#define EXPECT(cond) do { if (!(cond)) { std::printf("FAILED line %d: %s (P=%d T=%d G=%d grid=%d fold=%d)\n", __LINE__, #cond, P, T, G, grid, fold); return 1; } } while (0)

// Every unit is dealt to exactly one (CTA, slot); slots past a CTA's share are empty.
int check(int P, int T, int G, int grid, int fold) {
  const attn::UnitPlan plan = attn::unit_plan(P, T, G, fold);
  const int slots = attn::unit_slots(plan, static_cast<unsigned>(grid));
  std::vector<int> seen(static_cast<size_t>(P) * T, 0);
  for (int c = 0; c < grid; ++c)
    for (int s = 0; s < slots; ++s) {
      const int u = attn::unit_at(plan, static_cast<unsigned>(grid), static_cast<unsigned>(c), s);
      EXPECT(u >= -1 && u < P * T);
      if (u >= 0) EXPECT(seen[u]++ == 0);
    }
  for (int u = 0; u < P * T; ++u) EXPECT(seen[u] == 1);
  return 0;
}

// Causal weights (a query tile t of T sees T - t key tiles; the launch order
// puts t = 0 first): the heaviest CTA's total over the mean.
double imbalance(int P, int T, int G, int grid, int fold) {
  const attn::UnitPlan plan = attn::unit_plan(P, T, G, fold);
  const int slots = attn::unit_slots(plan, static_cast<unsigned>(grid));
  double total = 0.0, worst = 0.0;
  for (int c = 0; c < grid; ++c) {
    double load = 0.0;
    for (int s = 0; s < slots; ++s) {
      const int u = attn::unit_at(plan, static_cast<unsigned>(grid), static_cast<unsigned>(c), s);
      if (u < 0) continue;
      int p, t;
      attn::grouped_order(static_cast<unsigned>(u), P, T, G, &p, &t);
      load += T - t;
    }
    total += load;
    worst = std::max(worst, load);
  }
  return worst / (total / grid);
}

int main() {
  const int shapes[][2] = {{1, 1}, {1, 7}, {2, 1}, {3, 5}, {16, 128}, {37, 11}, {64, 3}, {5, 128}};
  const int grids[] = {1, 2, 3, 7, 148};
  for (const auto& sh : shapes)
    for (int G = 1; G <= sh[0]; G += (sh[0] > 8 ? 5 : 1))
      for (int grid : grids)
        for (int fold = 0; fold < 2; ++fold)
          if (check(sh[0], sh[1], G, grid, fold)) return 1;
  // The long-context causal grid (16 heads x 128 tiles, groups of 4 heads)
  // and a causal batch (128 problems x 32 tiles, groups of 16) on 148 CTAs:
  // folded pairs stay within 2 % of the mean, the plain snake does not.
  int P = 16, T = 128, G = 4, grid = 148, fold = 1;
  EXPECT(imbalance(P, T, G, grid, 1) < 1.02);
  EXPECT(imbalance(P, T, G, grid, 0) > 1.05);
  P = 128; T = 32; G = 16;
  EXPECT(imbalance(P, T, G, grid, 1) < 1.02);
  std::printf("ok\n");
  return 0;
}
"""


def test_persistent_plan_deals_every_unit_once_and_balances_causal_work(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no C++ compiler")
    src = tmp_path / "plan.cpp"
    src.write_text(PLAN_PROGRAM)
    exe = tmp_path / "plan"
    subprocess.run([cxx, "-std=c++17", "-O1", "-Wall", "-Wextra", "-Werror", "-I", CSRC, str(src), "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
