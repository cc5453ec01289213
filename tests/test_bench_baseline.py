"""bench.py's oracle baseline on the host (no GPU): the all-cores figure and
the same kind of sample on one thread, as the benchmark line reports them.
The oracle's OpenMP thread count is restored afterwards."""
import bench
import oracle
from workloads import TINY_F32, gen


def test_cpu_baseline_reports_all_cores_and_one_thread():
    w = TINY_F32.replace(per_token=False)
    qr = gen.make_queries(w, "cpu")["qr"]

    def kr_rows(n_docs):
        sub = w.replace(n_docs=n_docs, kv_on_host=False, per_token=False, n_needles=min(w.n_needles, n_docs))
        return gen.make_memory(sub, qr, "cpu")["kr_pool"]

    before = oracle.threads()
    b = bench.cpu_baseline(w, kr_rows, 0.2)
    assert oracle.threads() == before
    assert b["kind"] == "oracle" and b["unit"] == "tokens/s" and b["cores"] == before
    assert b["value"] > 0 and b["value_1thread"] > 0
    assert b["seconds_per_step"] > 0 and b["seconds_per_step_1thread"] > 0
    assert "one thread" in b["sample_1thread"]
    assert "cpu_model" in b
    short = bench.cpu_baseline(w, kr_rows, 0.2, one_thread=False)
    assert "value_1thread" not in short and short["value"] > 0


def test_interquartile_mean_drops_the_outer_quarters():
    assert bench.iq_mean([1.0, 2.0, 3.0, 4.0, 100.0]) == 3.0
    assert bench.iq_mean([5.0, 1.0, 9.0, 3.0, 7.0, 1000.0, -1000.0, 4.0]) == (3.0 + 4.0 + 5.0 + 7.0) / 4
    assert bench.iq_mean([2.5]) == 2.5


def test_decode_kernel_name_follows_the_plan_rule():
    from workloads import BY_NAME, TINY_F32
    assert bench.decode_kernel_name(BY_NAME["1m-bf16-4096x256-T64"]) == "decode_tc_kernel"
    assert bench.decode_kernel_name(BY_NAME["16m-bf16-lognormal-65536docs"]) == "decode_mma_kernel"
    assert bench.decode_kernel_name(TINY_F32) == "decode_kernel"
    bf = TINY_F32.replace(dtype="bf16", head_dim=128)
    assert bench.decode_kernel_name(bf.replace(n_q_heads=16, T=32)) == "decode_tc_kernel"   # G = 4, 128 rows
    assert bench.decode_kernel_name(bf.replace(n_q_heads=16, T=16)) == "decode_mma_kernel"  # 64 rows
    assert bench.decode_kernel_name(bf.replace(T=128)) == "decode_mma_kernel"               # G = 1


def test_decode_flops_count_visible_pairs():
    """4 d flops per visible (query row, key) pair, counted here by brute force:
    every memory key, and local key j for query token t when j <= L_b + t."""
    import numpy as np
    import torch
    from workloads import TINY_F32

    class BankStub:
        doc_chunk_off_host = torch.tensor([0, 3, 4, 9, 11])      # documents of 3, 1, 5, 2 chunks

    w = TINY_F32.replace(B=2, T=3, n_q_heads=8, n_kv_heads=4, head_dim=64)
    sel = np.array([[0, 2], [3, 1]])                             # 8 and 3 memory keys
    local_off = np.array([0, 10, 13])                            # live lengths 10 and 3 (L_b = 7 and 0)
    pairs = 0
    for b in range(w.B):
        n_mem = sum(int(BankStub.doc_chunk_off_host[d + 1] - BankStub.doc_chunk_off_host[d]) for d in sel[b])
        live = int(local_off[b + 1] - local_off[b])
        for t in range(w.T):
            for h in range(w.n_q_heads):
                pairs += n_mem + sum(1 for j in range(live) if j <= live - w.T + t)
    assert bench.decode_flops(w, BankStub, sel, local_off) == 4.0 * w.head_dim * pairs
