// Host-only check of the GEMM's stream-K work split (the same __host__
// __device__ functions the kernel uses).  Exit code 0 = all invariants hold.
//
//  1. CTA ranges [unit_begin(c), unit_begin(c+1)) are non-empty, ordered and
//     cover [0, units); unit_owner(u) is the CTA whose range holds u.
//  2. Every tile split between CTAs has a unique first contributor, so that
//     CTA index can key the tile's ticket.
//  3. The partial-slot rule agrees between writer and reducer: a CTA's
//     segment in tile t is its first segment iff unit_begin(c) >= t * ku.
//  4. The tail fast path (restating the kernel's prologue): a CTA whose last
//     segment is a split tile that it opens, with the next CTA as the only
//     other contributor, finds that CTA's share in its first-segment slot;
//     the head hand-off and the tail are different tiles; and the weight
//     producer's and the epilogue's notions of a split last segment agree.
#include <cstdio>
#include <cstdlib>
#include <set>

#include "gemm.cuh"

using qspec::unit_begin;
using qspec::unit_owner;

static int fail(const char* what, long long a, long long b, long long c) {
  std::printf("FAIL %s: %lld %lld %lld\n", what, a, b, c);
  return 1;
}

int main() {
  const long long grids[] = {1, 2, 3, 7, 64, 147, 148, 1024};
  const long long kus[] = {1, 2, 3, 32, 64, 86, 112, 224};
  const long long tiles_list[] = {1, 2, 3, 5, 32, 96, 172, 448, 7168};
  long long checked = 0;
  for (long long ku : kus) {
    for (long long tiles : tiles_list) {
      const long long units = ku * tiles;
      for (long long g0 : grids) {
        const long long grid = g0 < units ? g0 : units;
        // 1. partition
        if (unit_begin(0, units, grid) != 0 || unit_begin(grid, units, grid) != units)
          return fail("cover", units, grid, 0);
        for (long long c = 0; c < grid; ++c) {
          const long long b = unit_begin(c, units, grid), e = unit_begin(c + 1, units, grid);
          if (e <= b) return fail("empty range", units, grid, c);
          if (units <= 20000) {
            for (long long u = b; u < e; ++u)
              if (unit_owner(u, units, grid) != c) return fail("owner", units, grid, u);
          } else if (unit_owner(b, units, grid) != c || unit_owner(e - 1, units, grid) != c) {
            return fail("owner-ends", units, grid, c);
          }
        }
        // 2./3. split tiles
        std::set<long long> first_ctas;
        for (long long t = 0; t < tiles; ++t) {
          const long long t0 = t * ku;
          const long long lo = unit_owner(t0, units, grid);
          const long long hi = unit_owner(t0 + ku - 1, units, grid);
          if (lo == hi) continue;   // one CTA covers the whole tile: written directly
          if (!first_ctas.insert(lo).second) return fail("ticket collision", units, grid, t);
          for (long long c = lo; c <= hi; ++c) {
            const long long b = unit_begin(c, units, grid), e = unit_begin(c + 1, units, grid);
            const long long seg_start = b > t0 ? b : t0;
            if (seg_start >= (e < t0 + ku ? e : t0 + ku)) return fail("non-contributor", units, grid, c);
            const bool writer_first = (seg_start == b);
            const bool reducer_first = (b >= t0);
            if (writer_first != reducer_first) return fail("slot rule", units, grid, c);
          }
        }
        // 4. tail fast path and head hand-off, as the kernel computes them
        for (long long c = 0; c < grid; ++c) {
          const long long ub = unit_begin(c, units, grid), ue = unit_begin(c + 1, units, grid);
          const long long t_tail = (ue - 1) / ku, tail_u0 = t_tail * ku;
          const bool tail_split = !(ub <= tail_u0 && ue == tail_u0 + ku);
          const bool tail_fast =
              tail_split && ub <= tail_u0 && unit_owner(tail_u0 + ku - 1, units, grid) == c + 1;
          // the epilogue's last segment [max(ub, tail_u0), ue) and its "full" test
          const long long last_start = ub > tail_u0 ? ub : tail_u0;
          const bool last_full = (last_start == tail_u0) && (ue == tail_u0 + ku);
          if (last_full == tail_split) return fail("tail split rule", units, grid, c);
          if (tail_fast) {
            if (c + 1 >= grid) return fail("fast tail: no next CTA", units, grid, c);
            const long long nb = ue, ne = unit_begin(c + 2, units, grid);
            if (!(nb > tail_u0 && nb < tail_u0 + ku)) return fail("fast tail: next start", units, grid, c);
            if (ne < tail_u0 + ku) return fail("fast tail: next ends early", units, grid, c);
            // the next CTA's segment in the tile is its first one (slot 2 (c+1) + 0)
            if (!(nb >= tail_u0)) return fail("fast tail: slot", units, grid, c);
            if (unit_owner(tail_u0, units, grid) != c) return fail("fast tail: first contributor", units, grid, c);
          }
          const long long t_head = ub / ku, head_end = (ue < (t_head + 1) * ku) ? ue : (t_head + 1) * ku;
          const bool head_handoff = head_end < ue && ub != t_head * ku;
          if (head_handoff && tail_split && t_head == t_tail) return fail("head is tail", units, grid, c);
          if (head_handoff && (ue - ub) < 2) return fail("head hand-off in one unit", units, grid, c);
        }
        ++checked;
      }
    }
  }
  std::printf("ok %lld configurations\n", checked);
  return 0;
}
