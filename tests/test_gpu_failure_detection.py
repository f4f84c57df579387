"""Failure detection on the GPU without a fault: a bounded in-kernel wait on
an mbarrier phase that never completes gives up after its limit, records the
time-out in a word the host reads, and the kernel returns normally -- the CUDA
context stays usable for the next calls (the mechanism every pipeline wait of
the library uses, with its limit of one second)."""
import time

import pytest
import torch

import oracle
import synth
from bit_weight_streaming_dequant_b200 import q4dec
from gpu_util import assert_gemv_close, dev_bf16, dev_bytes

pytestmark = pytest.mark.gpu


def _selftest(limit_us, arrive):
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    st = q4dec.lib().q4d_wait_selftest(word.data_ptr(), limit_us, arrive,
                                       torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    return int(word.item()), time.perf_counter() - t0


def test_wait_that_never_completes_times_out_and_returns(cuda_ok):
    word, seconds = _selftest(50_000, arrive=0)   # 50 ms limit
    assert word == 1                              # the time-out bit, and not "completed"
    assert 0.045 <= seconds < 5.0


def test_wait_that_completes_reports_completion(cuda_ok):
    word, seconds = _selftest(5_000_000, arrive=1)
    assert word == 2 and seconds < 1.0


def test_context_usable_after_a_timed_out_wait(cuda_ok):
    assert _selftest(20_000, arrive=0)[0] == 1
    N, K, M = 300, 1280, 3
    W = synth.q4_0_weights(17, N, K)
    x = synth.activations(18, M, K)
    y = q4dec.q4_gemv(dev_bytes(W), dev_bf16(x), N=N, K=K)
    torch.cuda.synchronize()
    y_ref, S = oracle.gemv(W, x, M, N, K)
    assert_gemv_close(y, y_ref, S, "gemv after a timed-out wait")
    assert q4dec.device_error() == 0              # the library's own word is untouched
