"""Host-side check of how the single-launch kernel (csrc/fused_tc.cu) leaves
and merges the pieces of a segment spread over several CTAs.  The kernel's
own functions (between the ETA_PIECES markers: run_mode, piece_set_complete,
piece_announcement, piece_set) and the unit split it uses (UnitSplit from
attend_common.cuh) are compiled for the host with g++, inside a driver that
lays out segments of given unit counts, cuts the units into the kernel's
equal ranges [U c / N, U (c + 1) / N), forms each CTA's runs and modes the
way the kernel does, and applies the announcements of every shared segment
in several random orders.  It checks:

* every unit is covered once; a segment held by one CTA alone is written
  directly, any other leaves one piece per CTA whose range it touches;
* pieces never share a slot, and every piece but the first is in slot 0;
* exactly one announcement completes a segment's set, whatever the order,
  and it names the first and last CTAs, the first piece's slot, and a set
  of CTAs (those of the span with a non-empty range) equal to the pieces';
* ranges may be empty (fewer units than CTAs), a case the kernel once got
  wrong: a set then never completed."""
import os
import random
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "learned_threshold_sparse_b200", "csrc")


def _sources():
    common = open(os.path.join(CSRC, "attend_common.cuh")).read()
    m = re.search(r"struct UnitSplit \{.*?\n\};", common, flags=re.S)
    assert m, "UnitSplit not found"
    split = m.group(0).replace("__device__ __forceinline__", "inline")
    fused = open(os.path.join(CSRC, "fused_tc.cu")).read()
    m = re.search(r"// ETA_PIECES_BEGIN\n(.*?)// ETA_PIECES_END", fused, flags=re.S)
    assert m, "piece functions not found"
    return split, m.group(1).replace("__host__ __device__ inline", "inline")


DRIVER = r"""
#include <algorithm>
#include <cstdio>
#include <random>
#include <set>
#include <vector>
%s
%s
// stdin: scenarios "N S seed c_0 ... c_{S-1}" (units per segment), one per line.
// stdout: one line per scenario, "OK ..." or "FAIL reason".
int main() {
  int N, S;
  unsigned seed;
  while (scanf("%%d %%d %%u", &N, &S, &seed) == 3) {
    std::vector<long long> cnt(S), start(S + 1, 0);
    for (int g = 0; g < S; ++g) {
      scanf("%%lld", &cnt[g]);
      start[g + 1] = start[g] + cnt[g];
    }
    const long long U = start[S];
    UnitSplit us(static_cast<unsigned>(U), static_cast<unsigned>(N));
    std::vector<std::vector<std::pair<int, int>>> pieces(S);  // (cta, mode)
    std::vector<int> covered(S, 0);
    const char* fail = nullptr;
    for (int c = 0; c < N && !fail; ++c) {
      const long long u0 = us.start(c), u1 = us.start(c + 1);
      long long u = u0;
      int seg = 0;
      while (u < u1) {
        while (start[seg + 1] <= u) ++seg;
        const long long end = std::min(u1, start[seg + 1]);
        const bool holds_u0 = u == u0, at_u1 = end == u1;
        const bool shared_start = holds_u0 && start[seg] < u0;
        const bool shared_end = at_u1 && start[seg + 1] > u1;
        pieces[seg].push_back({c, run_mode(holds_u0, shared_start, shared_end)});
        covered[seg] += static_cast<int>(end - u);
        u = end;
      }
    }
    int shared_segs = 0, total_pieces = 0;
    for (int g = 0; g < S && !fail; ++g) {
      if (covered[g] != cnt[g]) { fail = "units not covered exactly once"; break; }
      const auto& pl = pieces[g];
      if (cnt[g] == 0) { if (!pl.empty()) fail = "a piece of an empty segment"; continue; }
      bool any_shared = false, all_shared = true;
      for (auto& p : pl) { any_shared |= (p.second & kModeShared) != 0; all_shared &= (p.second & kModeShared) != 0; }
      if (!any_shared) {
        if (pl.size() != 1 || pl[0].second != (kModeFirst | kModeLast)) fail = "a whole segment not written directly";
        continue;
      }
      if (!all_shared || pl.size() < 2) { fail = "a shared segment with an unshared or single piece"; break; }
      ++shared_segs;
      total_pieces += static_cast<int>(pl.size());
      std::set<int> slots, ctas;
      int firsts = 0, lasts = 0, first_cta = -1, first_slot = -1, last_cta = -1;
      for (auto& p : pl) {
        const int slot = 2 * p.first + ((p.second & kModeSlot1) ? 1 : 0);
        if (!slots.insert(slot).second) fail = "two pieces in one slot";
        ctas.insert(p.first);
        if (p.second & kModeFirst) { ++firsts; first_cta = p.first; first_slot = (p.second & kModeSlot1) ? 1 : 0; }
        else if (p.second & kModeSlot1) fail = "a piece after the first one outside slot 0";
        if (p.second & kModeLast) { ++lasts; last_cta = p.first; }
      }
      if (fail) break;
      if (firsts != 1 || lasts != 1) { fail = "not exactly one first and one last piece"; break; }
      std::mt19937 rng(seed + g);
      for (int rep = 0; rep < 6 && !fail; ++rep) {
        std::vector<std::pair<int, int>> order = pl;
        std::shuffle(order.begin(), order.end(), rng);
        unsigned long long v = 0;
        int completes = 0;
        for (auto& p : order) {
          v += piece_announcement(p.second, p.first);
          const PieceSet ps = piece_set(v);
          bool stale = false;
          if (!piece_set_complete(ps, us, N, &stale)) {
            if (stale) fail = "a live counter read as stale";
            continue;
          }
          std::set<int> span;
          for (int c = ps.c_first; c <= ps.c_last; ++c)
            if (us.owns_any(static_cast<unsigned>(c))) span.insert(c);
          ++completes;
          if (ps.c_first != first_cta || ps.c_last != last_cta) fail = "wrong first or last CTA";
          else if (ps.slot_first != first_slot) fail = "wrong slot of the first piece";
          else if (span != ctas) fail = "the span's CTAs differ from the pieces'";
        }
        if (!fail && completes != 1) fail = "the set did not complete exactly once";
      }
    }
    if (fail) printf("FAIL %%s\n", fail);
    else printf("OK %%d %%d\n", shared_segs, total_pieces);
  }
  return 0;
}
"""


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    d = tmp_path_factory.mktemp("pieces")
    prog = d / "pieces.cpp"
    prog.write_text(DRIVER % _sources())
    exe = d / "pieces"
    subprocess.run(["g++", "-O1", "-std=c++17", str(prog), "-o", str(exe)], check=True)

    def run(cases):
        text = "\n".join(f"{n} {len(c)} {seed} " + " ".join(str(x) for x in c) for n, c, seed in cases) + "\n"
        out = subprocess.run([str(exe)], input=text, capture_output=True, text=True, check=True).stdout.split("\n")
        return [ln for ln in out if ln]

    return run


def _check(lines):
    bad = [ln for ln in lines if not ln.startswith("OK")]
    assert not bad, bad[:5]
    return sum(int(ln.split()[1]) for ln in lines), sum(int(ln.split()[2]) for ln in lines)


def test_decode_workload_shapes(driver):
    # c3_long / c4_max (4 segments), c5_batched (32 ragged segments), c2_single
    cases = [(148, [777, 779, 781, 761], 1), (148, [1554, 1561, 1549, 1552], 2),
             (148, [300 + 40 * (k % 7) for k in range(32)], 3), (148, [195, 190, 201, 188], 4)]
    shared, pieces = _check(driver(cases))
    assert shared >= 36 and pieces >= 148  # every CTA holds a piece of some shared segment


def test_fewer_units_than_ctas(driver):
    cases = [(148, [26, 71], 5), (148, [1, 1, 1], 6), (300, [5, 0, 9, 0, 0, 2], 7), (7, [3], 8), (148, [0, 0, 0], 9)]
    _check(driver(cases))


@pytest.mark.parametrize("n", [1, 2, 3, 7, 148, 300])
def test_random_layouts(driver, n):
    rng = random.Random(n)
    cases = []
    for k in range(300):
        S = rng.randint(1, 40)
        kind = rng.random()
        if kind < 0.3:
            counts = [rng.choice([0, 0, 1, 2, 5]) for _ in range(S)]
        elif kind < 0.6:
            counts = [rng.randint(0, 3 * n) for _ in range(S)]
        else:
            counts = [rng.randint(0, 4000) for _ in range(S)]
        cases.append((n, counts, k))
    _check(driver(cases))


def _broken(tmp_path, name, old, new, scenario):
    split, pieces = _sources()
    broken = pieces.replace(old, new)
    assert broken != pieces
    prog = tmp_path / f"{name}.cpp"
    prog.write_text(DRIVER % (split, broken))
    exe = tmp_path / name
    subprocess.run(["g++", "-O1", "-std=c++17", str(prog), "-o", str(exe)], check=True)
    return subprocess.run([str(exe)], input=scenario, capture_output=True, text=True, check=True).stdout


def test_driver_sees_a_broken_slot_choice(tmp_path):
    out = _broken(tmp_path, "slot", "(holds_u0 ? 0 : kModeSlot1)", "(holds_u0 ? kModeSlot1 : 0)",
                  "148 4 1 777 779 781 761\n")
    assert out.startswith("FAIL"), out


def test_driver_sees_the_empty_range_bug(tmp_path):
    # counting every CTA of the span (empty ranges too) never completes a set
    # when there are fewer units than CTAs
    out = _broken(tmp_path, "span", "expect += us.owns_any(static_cast<unsigned>(c)) ? 1 : 0;", "expect += 1;",
                  "148 2 5 26 71\n")
    assert out.startswith("FAIL"), out
    assert _broken(tmp_path, "span2", "expect += us.owns_any(static_cast<unsigned>(c)) ? 1 : 0;", "expect += 1;",
                   "148 4 1 777 779 781 761\n").startswith("OK")
