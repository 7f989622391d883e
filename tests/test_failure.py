"""Failure detection without a GPU fault (needs a B200).

A kernel wait that can never complete gives up after its limit and reports
FA_ERR_TIMEOUT through fa_device_status; an out-of-range gather index is skipped and
reported as FA_ERR_INDEX. The context stays usable afterwards.
"""
import pytest
import torch

import tiled_exact_attention_fwd_b200 as fa

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from tiled_exact_attention_fwd_b200 import build
    build.build()
    fa.lib()
    fa.fa_device_status()  # clear anything earlier tests left


def test_bounded_wait_times_out_and_reports():
    fa.fa_selftest_bounded_wait(2_000_000)  # 2 ms
    st, where = fa.fa_device_status()
    assert st == -7 and where == 900
    assert fa.fa_device_status() == (0, 0)  # cleared
    # the context still works
    x = torch.ones(4, device="cuda:0")
    assert float((x * 2).sum()) == 8.0


def test_out_of_range_index_is_reported_and_skipped():
    dev = torch.device("cuda:0")
    x = torch.arange(4 * 16, dtype=torch.float32, device=dev).reshape(1, 4, 1, 16)
    idx = torch.tensor([1, 7], dtype=torch.int64, device=dev)
    u = fa.fa_unpad(x, idx)
    st, _ = fa.fa_device_status()
    assert st == -8
    assert torch.equal(u[0].cpu(), x[0, 1].cpu())
    assert float(u[1].abs().sum()) == 0.0


def test_status_waits_for_its_own_stream_only():
    import time
    a, b = torch.cuda.Stream(), torch.cuda.Stream()
    fa.fa_device_status(stream=a)  # first call: looks the error words up
    with torch.cuda.stream(b):
        torch.cuda._sleep(1_000_000_000)  # about half a second of GPU time on stream b
    t0 = time.perf_counter()
    st, _ = fa.fa_device_status(stream=a)
    dt = time.perf_counter() - t0
    b.synchronize()
    assert st == 0
    assert dt < 0.2, f"status on stream a waited {dt:.3f} s for stream b"
