"""Failure detection on the GPU without a fault: a bounded in-kernel wait on
a barrier that nothing completes runs out, records the timeout flag, and the
host reads it back as a status; the context stays usable afterwards."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import decoder_only_transformer_sdpa_b200 as A
    from workloads import random_qkv
    torch.cuda.set_device(0)
    assert A.attn_device_error() == 0
    A.attn_selftest_wait_timeout(4096)
    assert A.attn_device_error() == -6          # ATTN_ERR_TIMEOUT
    assert A.attn_device_error() == 0           # reading clears it
    inp = random_qkv(9, 1, 2, 130, 64, dtype=torch.bfloat16, do_std=1e-2)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, lse = A.attn_fwd(q, k, v)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    assert A.attn_device_error() == 0


def test_profile_hook_records_events():
    import decoder_only_transformer_sdpa_b200 as A
    from workloads import random_qkv
    inp = random_qkv(9, 2, 2, 256, 64, dtype=torch.bfloat16, do_std=1e-2)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    s = torch.cuda.current_stream()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in evs:
        e.record(s)
    A.attn_profile_next_call(evs[0], evs[1])
    o, lse = A.attn_fwd(q, k, v)
    assert A.attn_last_launch_count() == 1
    A.attn_profile_next_call(evs[2], evs[3])
    A.attn_bwd(q, k, v, o, lse, do)
    assert A.attn_last_launch_count() >= 1
    torch.cuda.synchronize()
    assert evs[0].elapsed_time(evs[1]) > 0 and evs[2].elapsed_time(evs[3]) > 0
