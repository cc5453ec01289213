"""The seeded synthetic inputs match the recipe the design states: document
counts, length distributions and their realised totals, local-context
lengths, and determinism.  Pure numpy on the host."""
import numpy as np
import oracle
from workloads import MEM_100M, MEM_16M, MEM_16M_B32, MEM_1M, gen


def _chunks(w):
    return int(oracle.chunk_offsets(gen.offsets(gen.doc_lengths(w)), w.chunk)[-1])


def test_fixed_length_memories():
    for w, docs, tokens in ((MEM_1M, 4096, 1 << 20), (MEM_100M, 390625, 100_000_000)):
        L = gen.doc_lengths(w)
        assert len(L) == docs and int(L.sum()) == tokens and np.all(L == 256)
        assert _chunks(w) == docs * 4
    assert _chunks(MEM_100M) == 1_562_500


def test_lognormal_16m_memory():
    L = gen.doc_lengths(MEM_16M)
    assert len(L) == 65536
    assert L.min() >= 32 and L.max() <= 4096
    assert abs(float(np.median(L)) - 256) <= 4                  # median 256
    s = float(np.std(np.log(L)))
    assert 0.28 < s < 0.32                                       # sigma 0.3 (clipping is rare)
    assert int(L.sum()) == 17_542_667                           # 17.54M tokens (reported)
    assert _chunks(MEM_16M) == 306_369
    assert np.array_equal(L, gen.doc_lengths(MEM_16M))            # seeded: the same every call
    assert np.array_equal(gen.doc_lengths(MEM_16M_B32), L)       # the batch shares the memory


def test_batch_local_contexts():
    lens = gen.local_lengths(MEM_16M_B32)
    assert len(lens) == 32 and lens.min() >= 1024 and lens.max() <= 8192
    assert np.array_equal(lens, gen.local_lengths(MEM_16M_B32))
    assert np.all(gen.local_lengths(MEM_16M) == gen.local_lengths(MEM_16M)[0])
