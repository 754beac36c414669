"""Failure detection on the GPU without a fault: a bounded wait that can never
complete gives up, the host reads the timeout from the device error word, and
the context stays usable for the next launch."""
import time

import pytest

import oracle
from h3_testlib import bf16_bits_to_f64, check_attention, from_cuda_bf16, to_cuda_bf16
from video_diffusion_transformer_h3attn_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h3():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import video_diffusion_transformer_h3attn_b200 as mod
    return mod


def test_bounded_wait_times_out_and_is_reported(h3):
    h3.device_status()  # start from a clear error word
    t0 = time.perf_counter()
    h3.selftest_wait_timeout()
    with pytest.raises(h3.H3AttnError, match="timed out") as exc:
        h3.device_status()
    elapsed = time.perf_counter() - t0
    assert exc.value.status == 5, "expected H3ATTN_ERR_DEVICE_TIMEOUT"
    assert 0.5 < elapsed < 30.0, "the wait bound is about one second (took %.2f s)" % elapsed
    h3.device_status()  # the previous call cleared the word
    # the context is still usable: a small attention call matches the oracle
    w = inputs.random_case([300], 2, 128, seed=4242)
    o, lse = h3.attention(to_cuda_bf16(w.q), to_cuda_bf16(w.k), to_cuda_bf16(w.v), return_lse=True)
    h3.device_status()
    ro, rl = oracle.get().attention(w.q, w.k, w.v, w.cu_seqlens)
    check_attention(bf16_bits_to_f64(from_cuda_bf16(o)), ro, "after a timeout", lse.cpu().numpy().T, rl,
                    strict=True)
