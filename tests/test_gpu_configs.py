"""The workloads at full size, in the launch configuration bench.py times, checked against the
oracle: every sequence of the 1M-context Reindex and the Minimal workloads, 16 sequences spread over
the batch of the 131,072-context Full workload, 72 query rows of the prefill chunk (its first and
last rows among them) and every row of 16 sequences of the multi-token decode: index sets and pools
identical, attention within tolerance. The oracle runs in spawned host processes (the sequences of
the 131,072-context workloads and the 1M-position prefill cache take tens of seconds each to build
on the host, which bounds how many of them fit in a test run)."""
import numpy as np
import pytest
import torch

from _oracle_pool import oracle_steps
from workloads import gpu as G

pytestmark = pytest.mark.gpu

CASES = [
    ("full_b1_n4096", [0]),
    ("full_b64_n131072", list(range(0, 64, 4)) + [63]),
    ("reindex_b128_n1m", list(range(128))),
    ("minimal_b256_n262144", list(range(256))),
]


def _cmp_attn(out, of, ro, tol=2e-3):
    assert torch.equal(out, of.to(torch.bfloat16))
    err = np.abs(of.double().cpu().numpy() - ro).max()
    assert err <= tol, err


@pytest.mark.parametrize("name,seqs", CASES)
def test_decode_workload_sampled(orc, name, seqs):
    step = G.build(name)
    of = torch.empty(step.batch, 16, 128, dtype=torch.float32, device="cuda")
    step.run(out_f32=of)
    import compressed_sparse_attention_append_b200 as csa

    assert csa.csa2_get_device_status(step.ws) == 0
    wl = step.wl
    ref = oracle_steps(name, seqs)
    for b in seqs:
        r = ref[b]
        if wl.mode != "minimal":
            assert np.array_equal(step.outputs["idx"][b].cpu().numpy(), r["idx"]), b
        if wl.mode == "full" and wl.pool_blocks:
            assert np.array_equal(step.outputs["pool"][b].cpu().numpy(), r["pool"])
            assert int(step.outputs["pool_n"][b]) == r["pool_n"]
        _cmp_attn(step.outputs["out"][b], of[b], r["out"])
    # a second step on the same state gives the same result (counters cleared, appends idempotent)
    prev = {k: v.clone() for k, v in step.outputs.items()}
    step.run()
    for k, v in step.outputs.items():
        assert torch.equal(v, prev[k]), k
    del step
    torch.cuda.empty_cache()


def test_prefill_workload_sampled_rows(orc):
    name = "prefill_t4096_at_1m"
    step = G.build(name)
    wl = step.wl
    of = torch.empty(wl.tq, 16, 128, dtype=torch.float32, device="cuda")
    step.run(out_f32=of)
    torch.cuda.synchronize()
    rows = sorted(set([0, 1, 2, 3, 2047, 4094, 4095] + list(range(5, 4096, 63))))
    assert len(rows) >= 64
    groups = [rows[j::8] for j in range(8)]  # each process builds the 1M-position cache once
    r = oracle_steps(name, [0], rows=groups)[0]
    for i in rows:
        idx, ro, _ = r["rows"][i]
        assert np.array_equal(step.outputs["idx"][i].cpu().numpy(), idx), i
        _cmp_attn(step.outputs["out"][i], of[i], ro)
    del step
    torch.cuda.empty_cache()


def test_draft_workload_sampled(orc):
    """Multi-token decode (5 draft tokens per sequence, 64 sequences at N = 131,072): the three calls
    bench.py times; every row of 17 sequences spread over the batch against the oracle."""
    import compressed_sparse_attention_append_b200 as csa

    step = G.build("draft_b64_n131072_tq5")
    wl = step.wl
    of = torch.empty(step.batch, wl.tq, 16, 128, dtype=torch.float32, device="cuda")
    step.run(out_f32=of)
    assert csa.csa2_get_device_status(step.ws) == 0
    seqs = list(range(0, step.batch, 4)) + [step.batch - 1]
    ref = oracle_steps("draft_b64_n131072_tq5", seqs)
    for b in seqs:
        r = ref[b]
        for t in range(wl.tq):
            idx, ro, _ = r["rows"][t]
            assert np.array_equal(step.outputs["idx"][b, t].cpu().numpy(), idx), (b, t)
            _cmp_attn(step.outputs["out"][b, t], of[b, t], ro)
    prev = {k: v.clone() for k, v in step.outputs.items()}
    step.run()
    for k, v in step.outputs.items():
        assert torch.equal(v, prev[k]), k
    del step
    torch.cuda.empty_cache()
