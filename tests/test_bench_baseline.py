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
