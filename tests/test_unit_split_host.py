"""Host-side check of the work split the persistent attention kernel and the
merge kernel share: the UnitSplit code from attend_common.cuh is compiled for
the host (device qualifiers replaced by `inline`) and, over many unit counts
U and grid sizes N, must give the ranges [floor(U c / N), floor(U (c + 1) / N))
exactly (32-bit arithmetic included), and owner(u) must name the range that
holds u.  A wrong owner would send the merge to the wrong partial slots."""
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "learned_threshold_sparse_b200", "csrc", "attend_common.cuh")

US = [0, 1, 2, 3, 5, 147, 148, 149, 295, 296, 297, 1000, 3098, 6216, 16384, 65537, 262144, 1 << 20, 10_000_019]
NS = [1, 2, 3, 7, 148, 296, 592]


def _struct_source():
    src = open(HEADER).read()
    m = re.search(r"struct UnitSplit \{.*?\n\};", src, flags=re.S)
    assert m, "UnitSplit not found"
    return m.group(0).replace("__device__ __forceinline__", "inline")


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    d = tmp_path_factory.mktemp("split")
    prog = d / "split.cpp"
    prog.write_text("\n".join([
        "#include <cstdio>",
        "#include <cstdlib>",
        _struct_source(),
        "int main(int argc, char** argv) {",
        "  const unsigned U = strtoul(argv[1], 0, 10), N = strtoul(argv[2], 0, 10);",
        "  UnitSplit s(U, N);",
        "  for (unsigned c = 0; c <= N; ++c) printf(\"S %u %u\\n\", c, s.start(c));",
        "  for (unsigned c = 0; c < N; ++c) printf(\"A %u %d\\n\", c, s.owns_any(c) ? 1 : 0);",
        "  const unsigned step = U > 200000 ? U / 200000 : 1;",
        "  for (unsigned u = 0; u < U; u += step) printf(\"O %u %u\\n\", u, s.owner(u));",
        "  if (U > 0) printf(\"O %u %u\\n\", U - 1, s.owner(U - 1));",
        "  return 0;",
        "}",
    ]))
    exe = d / "split"
    subprocess.run(["g++", "-O1", "-std=c++17", str(prog), "-o", str(exe)], check=True)
    return str(exe)


@pytest.mark.parametrize("N", NS)
@pytest.mark.parametrize("U", US)
def test_split_ranges_and_owner(probe, U, N):
    out = subprocess.run([probe, str(U), str(N)], capture_output=True, text=True, check=True).stdout.split("\n")
    start, any_, owner = {}, {}, {}
    for ln in out:
        if not ln:
            continue
        k, a, b = ln.split()
        {"S": start, "A": any_, "O": owner}[k][int(a)] = int(b)
    for c in range(N + 1):
        assert start[c] == U * c // N, (c, start[c])
    for c in range(N):
        assert any_[c] == (1 if start[c + 1] > start[c] else 0)
    for u, c in owner.items():
        assert start[c] <= u < start[c + 1], (u, c, start[c], start[c + 1])
