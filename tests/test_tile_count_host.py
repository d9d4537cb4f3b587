"""Host-side check of count_tiles (attend_common.cuh): the MMA and softmax
warps of the tensor-core attention kernel learn from it how many tiles their
producer will issue for the CTA's unit range, so it must agree with the
producer's packing rule (consecutive units of one segment, BPT to a tile, a
tile never crossing a segment boundary) for every range of the work split.
The function is compiled for the host from the kernel header (device
qualifiers replaced by `inline`, Shape reduced to the two fields it reads)."""
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "learned_threshold_sparse_b200", "csrc", "attend_common.cuh")


def _count_tiles_source():
    src = open(HEADER).read()
    m = re.search(r"template <int BPT>\n__device__ __forceinline__ int count_tiles\(.*?\n  return tiles;\n\}", src,
                  flags=re.S)
    assert m, "count_tiles not found"
    return m.group(0).replace("__device__ __forceinline__", "inline")


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    d = tmp_path_factory.mktemp("tiles")
    prog = d / "tiles.cpp"
    prog.write_text("\n".join([
        "#include <algorithm>",
        "#include <cstdio>",
        "#include <vector>",
        "using std::max; using std::min;",
        "struct Shape { int nseg, nchunks; };",
        _count_tiles_source(),
        "int main() {",
        "  Shape s; int N;",
        "  if (scanf(\"%d %d %d\", &s.nseg, &s.nchunks, &N) != 3) return 1;",
        "  const int n = s.nseg * s.nchunks;",
        "  std::vector<int> prefix(n + 1);",
        "  for (int i = 0; i <= n; ++i)",
        "    if (scanf(\"%d\", &prefix[i]) != 1) return 1;",
        "  const long long U = prefix[n];",
        "  for (int c = 0; c < N; ++c) {",
        "    const int u0 = (int)(U * c / N), u1 = (int)(U * (c + 1) / N);",
        "    printf(\"%d %d %d %d\\n\", u0, u1, count_tiles<1>(prefix.data(), s, u0, u1),",
        "           count_tiles<2>(prefix.data(), s, u0, u1));",
        "  }",
        "  return 0;",
        "}",
    ]))
    exe = d / "tiles"
    subprocess.run(["g++", "-O1", "-std=c++17", str(prog), "-o", str(exe)], check=True)
    return str(exe)


def _producer_tiles(seg_of_unit, u0, u1, bpt):
    """Tiles the producer emits for units [u0, u1): a pending tile goes out
    when the next unit belongs to another segment or when it holds bpt units,
    and the last one at the end of the range."""
    tiles, pend, pend_seg = 0, 0, None
    for u in range(u0, u1):
        sg = seg_of_unit[u]
        if pend and sg != pend_seg:
            tiles += 1
            pend = 0
        if not pend:
            pend_seg = sg
        pend += 1
        if pend == bpt:
            tiles += 1
            pend = 0
    return tiles + (1 if pend else 0)


@pytest.mark.parametrize("nseg,nchunks,chunk,N,density,seed", [
    (1, 64, 64, 148, 0.38, 0), (4, 64, 32, 148, 0.38, 1), (4, 128, 64, 148, 0.17, 2),
    (32, 8, 256, 148, 0.64, 3), (8, 16, 64, 296, 0.05, 4), (4, 32, 64, 148, 0.0, 5),
    (2, 4, 32, 148, 1.0, 6), (16, 64, 32, 7, 0.5, 7), (3, 5, 32, 1, 0.3, 8),
])
def test_count_tiles_matches_producer(probe, nseg, nchunks, chunk, N, density, seed):
    rng = np.random.default_rng(seed)
    counts = rng.binomial(chunk, density, size=nseg * nchunks)
    # whole empty segments and empty chunks occur in ragged batches
    counts[rng.random(counts.size) < 0.1] = 0
    if nseg > 2:
        counts[nchunks:2 * nchunks] = 0
    prefix = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    seg_of_unit = np.repeat(np.arange(nseg), [int(counts[s * nchunks:(s + 1) * nchunks].sum()) for s in range(nseg)])
    inp = f"{nseg} {nchunks} {N}\n" + " ".join(str(int(x)) for x in prefix) + "\n"
    out = subprocess.run([probe], input=inp, capture_output=True, text=True, check=True).stdout.split("\n")
    rows = [list(map(int, ln.split())) for ln in out if ln.strip()]
    assert len(rows) == N
    for u0, u1, t1, t2 in rows:
        assert t1 == _producer_tiles(seg_of_unit, u0, u1, 1), (u0, u1)
        assert t2 == _producer_tiles(seg_of_unit, u0, u1, 2), (u0, u1)
