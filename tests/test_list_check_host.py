"""Host-side check of the consistency predicates the attention walkers apply
to the screen's chunk tables before they stream a row (attend_common.cuh,
between the ETA_LIST_CHECK markers).  The predicates are compiled for the
host with g++ (device qualifiers replaced by `inline`) inside a small driver
that walks a table the way the warp walker does: per chunk the count, then
every entry against the one before it.

Valid tables are built from the oracle's admitted sets (per query head,
section 3.1 screen with the always-loaded window and the top-1 rescue of
Appendix F.4): the union of a KV group's heads, ascending, with a G-bit head
mask per block.  They must pass untouched, including ragged last chunks and
lengths that end inside a block.  Each corruption a stale or overwritten
table can show (a count above the chunk or below zero, a block from another
chunk or past the sequence, a repeated or descending block, an empty mask or
a mask bit beyond the group) must raise its own fault bit."""
import os
import re
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "learned_threshold_sparse_b200", "csrc", "attend_common.cuh")

F_COUNT, F_BLOCK, F_ORDER, F_MASK = 1, 2, 4, 8


def _check_source():
    src = open(HEADER).read()
    m = re.search(r"// ETA_LIST_CHECK_BEGIN\n(.*?)// ETA_LIST_CHECK_END", src, flags=re.S)
    assert m, "list check block not found"
    return m.group(1).replace("__host__ __device__ __forceinline__", "inline")


DRIVER = r"""
#include <cstdio>
%s
// stdin: chunk G T b nchunks, then per chunk: count and `count` entries.
// stdout: per chunk the OR of its fault bits.
int main() {
  int chunk, G, T, b, nchunks;
  if (scanf("%%d %%d %%d %%d %%d", &chunk, &G, &T, &b, &nchunks) != 5) return 2;
  const int nblocks = (T + b - 1) / b;
  for (int c = 0; c < nchunks; ++c) {
    int count;
    if (scanf("%%d", &count) != 1) return 3;
    unsigned f = chunk_count_faults(chunk, count);
    int prev = -1;
    for (int k = 0; k < count; ++k) {
      long long e;
      if (scanf("%%lld", &e) != 1) return 4;
      const int entry = static_cast<int>(static_cast<unsigned>(e));
      f |= list_entry_faults(chunk, G, nblocks, c, entry, prev);
      prev = entry & ((1 << 24) - 1);
    }
    printf("%%u\n", f);
  }
  return 0;
}
"""


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    d = tmp_path_factory.mktemp("listcheck")
    prog = d / "listcheck.cpp"
    prog.write_text(DRIVER % _check_source())
    exe = d / "listcheck"
    subprocess.run(["g++", "-O1", "-std=c++17", str(prog), "-o", str(exe)], check=True)

    def run(chunk, G, T, b, tables):
        lines = [f"{chunk} {G} {T} {b} {len(tables)}"]
        for entries in tables:
            lines.append(" ".join(str(x) for x in [len(entries)] + [int(e) & 0xFFFFFFFF for e in entries]))
        out = subprocess.run([str(exe)], input="\n".join(lines) + "\n", capture_output=True, text=True, check=True)
        return [int(x) for x in out.stdout.split()]

    def run_counts(chunk, G, T, b, counts_and_entries):
        # a count that differs from the number of entries given (negative counts carry none)
        lines = [f"{chunk} {G} {T} {b} {len(counts_and_entries)}"]
        for count, entries in counts_and_entries:
            lines.append(" ".join(str(x) for x in [count] + [int(e) & 0xFFFFFFFF for e in entries]))
        out = subprocess.run([str(exe)], input="\n".join(lines) + "\n", capture_output=True, text=True, check=True)
        return [int(x) for x in out.stdout.split()]

    run.counts = run_counts
    return run


def entry(blk, mask):
    return blk | (mask << 24)


def valid_tables(rng, T, b, G, chunk, n_local_blocks, density):
    """Chunk tables of one KV group, built from the oracle's per-head
    admitted sets on random block scores."""
    nb = -(-T // b)
    adm = np.zeros((G, nb), bool)
    for h in range(G):
        scores = rng.standard_normal(nb)
        tau = np.quantile(scores, 1.0 - density) if nb else 0.0
        adm[h], _ = oracle.admit(scores, float(tau), nb, n_local_blocks)
    nchunks = -(-nb // chunk)
    tables = []
    for c in range(nchunks):
        ent = []
        for blk in range(c * chunk, min(nb, (c + 1) * chunk)):
            mask = int(sum(1 << h for h in range(G) if adm[h, blk]))
            if mask:
                ent.append(entry(blk, mask))
        tables.append(ent)
    return tables


CASES = [  # T, b, G, chunk, n_local_blocks, density
    (4096, 64, 1, 16, 2, 0.3),
    (32768, 64, 4, 64, 2, 0.2),
    (1000, 64, 8, 4, 2, 0.5),
    (130, 16, 2, 3, 0, 0.05),
    (65, 64, 4, 8, -1, 0.0),   # rescue only: one block per head
    (524288, 128, 4, 256, 2, 0.17),
    (64, 64, 8, 16, 2, 1.0),
]


@pytest.mark.parametrize("case", CASES)
def test_screen_tables_pass(checker, case):
    T, b, G, chunk, nl, dens = case
    rng = np.random.default_rng(T + G)
    tables = valid_tables(rng, T, b, G, chunk, nl, dens)
    assert sum(len(t) for t in tables) > 0
    assert checker(chunk, G, T, b, tables) == [0] * len(tables)


def test_empty_and_full_chunks_pass(checker):
    chunk, G, T, b = 8, 4, 8 * 64 * 3 - 10, 64  # last chunk ragged, last block partial
    full = [[entry(c * chunk + j, 0xF) for j in range(chunk)] for c in range(3)]
    full[2] = full[2][:chunk]  # blocks 16..23, the sequence has 24 blocks
    assert checker(chunk, G, T, b, full) == [0, 0, 0]
    assert checker(chunk, G, T, b, [[], [], []]) == [0, 0, 0]


@pytest.fixture
def base():
    chunk, G, T, b = 8, 4, 8 * 64 * 2 + 40, 64  # 17 blocks (the last one partial): chunks [0,8) [8,16) [16,17)
    tables = [[entry(0, 1), entry(3, 0b0110), entry(7, 0b1000)],
              [entry(8, 0b1111), entry(12, 0b0001)],
              [entry(16, 0b0010)]]
    return chunk, G, T, b, tables


def test_base_table_passes(checker, base):
    chunk, G, T, b, tables = base
    assert checker(chunk, G, T, b, tables) == [0, 0, 0]


@pytest.mark.parametrize("mutate,chunk_idx,bit", [
    (lambda t: t[0].__setitem__(1, entry(9, 0b0110)), 0, F_BLOCK | F_ORDER),  # block of the next chunk; the 7 after it descends
    (lambda t: t[1].__setitem__(0, entry(7, 0b1111)), 1, F_BLOCK),             # block of the previous chunk
    (lambda t: t[2].__setitem__(0, entry(17, 0b0010)), 2, F_BLOCK),            # past the last block of the sequence
    (lambda t: t[2].__setitem__(0, entry(23, 0b0010)), 2, F_BLOCK),            # inside the chunk's span, past the sequence
    (lambda t: t[0].__setitem__(2, entry(3, 0b1000)), 0, F_ORDER),             # repeated block
    (lambda t: t[0].__setitem__(1, entry(0, 0b0110)), 0, F_ORDER),             # repeated first block
    (lambda t: t[1].reverse(), 1, F_ORDER),                                    # descending
    (lambda t: t[0].__setitem__(1, entry(3, 0)), 0, F_MASK),                   # empty head mask
    (lambda t: t[0].__setitem__(1, entry(3, 0b10000)), 0, F_MASK),             # head bit G (group of 4)
    (lambda t: t[1].__setitem__(1, 0x7F7F7F7F), 1, F_BLOCK | F_MASK),          # stale fill byte pattern
    (lambda t: t[1].__setitem__(1, -1), 1, F_BLOCK | F_MASK),                  # all bits set
])
def test_each_corruption_raises_its_fault(checker, base, mutate, chunk_idx, bit):
    chunk, G, T, b, tables = base
    tables = [list(t) for t in tables]
    mutate(tables)
    got = checker(chunk, G, T, b, tables)
    want = [0, 0, 0]
    want[chunk_idx] = bit
    assert got == want


def test_bad_counts(checker, base):
    chunk, G, T, b, tables = base
    over = [(chunk + 1, [entry(j, 1) for j in range(chunk + 1)]), (len(tables[1]), tables[1]), (1, tables[2])]
    assert checker.counts(chunk, G, T, b, over)[0] & F_COUNT
    neg = [(-1, []), (len(tables[1]), tables[1]), (1, tables[2])]
    assert checker.counts(chunk, G, T, b, neg) == [F_COUNT, 0, 0]
    exact = [(chunk, [entry(j, 1) for j in range(chunk)]), (0, []), (0, [])]
    assert checker.counts(chunk, G, T, b, exact) == [0, 0, 0]


def test_zero_length_sequence_admits_nothing(checker):
    assert checker(4, 2, 0, 64, [[entry(0, 1)]]) == [F_BLOCK]
    assert checker(4, 2, 0, 64, [[]]) == [0]


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_mask_width_follows_group(checker, G):
    chunk, T, b = 4, 256, 64
    ok = [[entry(0, (1 << G) - 1), entry(1, 1 << (G - 1))]]
    assert checker(chunk, G, T, b, ok) == [0]
    if G < 8:
        assert checker(chunk, G, T, b, [[entry(0, 1 << G)]]) == [F_MASK]
