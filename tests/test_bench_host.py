"""Host-side logic of bench.py that needs no GPU: which workloads' steps run
as one fused decode launch (pkv_paged_attn_decode_append appends exactly one
row per request, at position kv_lens - 1)."""
import numpy as np
import pytest

import bench
from workloads import make_workload


@pytest.mark.parametrize("name,kw", [("tiny_decode", {}), ("qwen3_decode", {"B": 8}),
                                     ("splitk_long", {"lens": [4000, 33]}),
                                     ("frag_large", {"B": 24, "median": 300.0, "max_len": 2000})])
def test_decode_only_steps_fuse(name, kw):
    w = make_workload(name, 0, **kw)
    _, _, slots = w.batch_new()
    assert bench.fusable_decode_step(w, slots)
    # one wrong slot (a row that is not its request's last position) and the
    # step must keep its separate append
    bad = np.array(slots, copy=True)
    bad[-1] = bad[-1] - 1 if bad[-1] > 0 else bad[-1] + 1
    assert not bench.fusable_decode_step(w, bad)
    assert not bench.fusable_decode_step(w, slots[:-1])


@pytest.mark.parametrize("name", ["mixed_prefill_decode", "spec_verify"])
def test_steps_with_chunks_do_not_fuse(name):
    w = make_workload(name, 0)
    _, _, slots = w.batch_new()
    assert not bench.fusable_decode_step(w, slots)
