"""Two host threads calling the library at once on one device, each with its
own stream, inputs and workspace: the kernels' shared-memory opt-in is set
once per (device, kernel) under a lock, and the per-call state (launch
counts, problem descriptions) is private to each call, so both threads'
results must match the oracle."""
import threading

import numpy as np
import pytest

from _helpers import LSE_MAX_ABS, assert_close_bf16, lse_err, to_dev, to_np
from exact_io_aware_45_b200 import fa, inputs
from oracle import attention as orc

pytestmark = pytest.mark.gpu


def test_two_host_threads_one_device():
    import torch
    fa.lib()
    cases = [(1, 4, 2, 384, 128, True, 41), (2, 2, 2, 300, 64, False, 42)]
    results, errors = {}, []
    start = threading.Barrier(len(cases))

    def worker(idx, case):
        try:
            B, Hq, Hkv, N, d, causal, seed = case
            torch.cuda.set_device(0)
            x = inputs.random_case(B, Hq, Hkv, N, d, seed=seed)
            stream = torch.cuda.Stream()
            with torch.cuda.stream(stream):
                q, k, v, do = (to_dev(x[n], torch.bfloat16) for n in ("q", "k", "v", "do"))
                scale = 1.0 / np.sqrt(d)
                start.wait()
                for _ in range(5):
                    o, lse = fa.forward(q, k, v, scale, causal)
                    dq, dk, dv = fa.backward(q, k, v, o, do, lse, scale, causal)
            stream.synchronize()
            results[idx] = (x, scale, causal, o, lse, dq, dk, dv)
        except Exception as e:  # reported below, on the main thread
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(i, c)) for i, c in enumerate(cases)]
    for th in threads:
        th.start()
    for th in threads:
        th.join(timeout=300)
    assert not errors, errors
    assert len(results) == len(cases)
    for x, scale, causal, o, lse, dq, dk, dv in results.values():
        O, L = orc.forward(x["q"], x["k"], x["v"], scale, causal)
        assert_close_bf16("O", to_np(o), O)
        assert lse_err(to_np(lse), L) <= LSE_MAX_ABS
        dQ, dK, dV = orc.backward(x["q"], x["k"], x["v"], x["do"], scale, causal, O=O)
        assert_close_bf16("dQ", to_np(dq), dQ)
        assert_close_bf16("dK", to_np(dk), dK)
        assert_close_bf16("dV", to_np(dv), dV)
