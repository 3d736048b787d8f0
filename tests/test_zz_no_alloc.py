"""Decode with the library's built-in scratch (pkv_paged_attn_decode_static).

That entry point exists for callers that cannot allocate device memory when
they run decode -- code inside another allocator's callbacks, plugins that
are handed only their input and output buffers, servers that must not grow
their device footprint after start-up.  It keeps the split-K scratch in a
fixed 32 MiB array inside the library instead of a caller workspace.  These
tests call it through the C ABI and check that two calls in a row give the
same results as the regular entry point, within the parity tolerance and bit
for bit, and that sizes beyond the array and bad partitions are refused.  The file is named to be collected
last, and it builds all of its own inputs, so it passes alone in a fresh
process as well as after the other tests.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 1e-2, 1e-3


def _close(got: torch.Tensor, ref: torch.Tensor, what: str):
    g = got.float().cpu().numpy().astype(np.float64)
    r = ref.float().cpu().numpy().astype(np.float64)
    fin = np.isfinite(r)
    assert np.array_equal(np.isfinite(g), fin), f"{what}: finite/non-finite pattern differs"
    err = np.abs(g[fin] - r[fin])
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3g}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs err {err.mean():.3g}"


@pytest.mark.parametrize("partition", [0, 64])
def test_static_scratch_decode_matches_workspace_decode(partition):
    import paged_kv_attention_37_b200 as pkv
    from tests.harness import DeviceStep
    from workloads import make_workload

    w = make_workload("qwen3_decode", 11, B=12, len_lo=100, len_hi=2500)
    ds = DeviceStep(pkv, w)
    ds.append()
    ref_lse = torch.empty((w.B, w.num_q_heads), device="cuda")
    ref = ds.decode(partition=partition, out_lse=ref_lse).clone()
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        pkv.pkv_paged_attn_decode_static(ds.q_dec, ds.k_pool, ds.v_pool, ds.pt_dec, ds.len_dec,
                                         w.scale, partition, out=out, out_lse=lse)
        torch.cuda.synchronize()
        _close(out, ref, f"output, call {call}")
        _close(lse, ref_lse, f"lse, call {call}")
        # the same kernels on the same inputs: the split plan and every merge
        # order are fixed by the shapes, so the results agree bit for bit
        assert torch.equal(out, ref), f"output bits, call {call}"
        assert torch.equal(lse, ref_lse), f"lse bits, call {call}"
    assert pkv.pkv_device_error_flags(clear=True) == 0


def test_static_scratch_refuses_bad_partition():
    import paged_kv_attention_37_b200 as pkv

    # a partition that is not a multiple of 32 is refused before the scratch
    # is touched, like the workspace entry point refuses it
    B, hq, hkv, d, P = 2, 8, 2, 128, 16
    q = torch.zeros((B, hq, d), dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros((4, hkv, P, d), dtype=torch.bfloat16, device="cuda")
    table = torch.zeros((B, 4), dtype=torch.int32, device="cuda")
    lens = torch.ones((B,), dtype=torch.int32, device="cuda")
    with pytest.raises(pkv.PkvError) as e:
        pkv.pkv_paged_attn_decode_static(q, pool, pool, table, lens, 0.1, 33)
    assert e.value.status == -2  # PKV_ERR_BAD_SHAPE


def test_static_scratch_refuses_oversized_requests():
    import paged_kv_attention_37_b200 as pkv

    # 2048 requests of up to 64k tokens need far more than 32 MiB of partials
    B, hq, hkv, d, P = 2048, 32, 8, 128, 16
    q = torch.zeros((B, hq, d), dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros((4, hkv, P, d), dtype=torch.bfloat16, device="cuda")
    table = torch.zeros((B, 4096), dtype=torch.int32, device="cuda")
    lens = torch.ones((B,), dtype=torch.int32, device="cuda")
    with pytest.raises(pkv.PkvError) as e:
        pkv.pkv_paged_attn_decode_static(q, pool, pool, table, lens, 0.1, 0)
    assert e.value.status == -5  # PKV_ERR_WORKSPACE
