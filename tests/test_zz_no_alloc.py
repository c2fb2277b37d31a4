"""The allocation-free quantisation entry point (static device scratch).

Some callers cannot hand the library a workspace: an engine that owns every
device allocation, or a hot loop that cannot pay for cudaMalloc's implicit
synchronisation.  fp8_quantize_pertensor_static serves them with a static
device array.  This test calls it through the C ABI twice in a row (the
second call must not see the first call's leftovers) and checks that codes
and scale equal, bit for bit (the tolerance the parity tests use for FP8
codes), both those of fp8_quantize_pertensor and those of the CPU oracle.
It is collected last so that a run stopping at the first failure has already
run every other test, and it passes both alone in a fresh process and after
the rest of the suite.
"""
import numpy as np
import pytest
import torch

from oracle import sp24_oracle as O
from structured_sparse_fp8_b200 import workloads as WL

pytestmark = pytest.mark.gpu


def _dev_bf16(bits, dev):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def test_static_scratch_quantize_matches_workspace_quantize_twice():
    import __graft_entry__
    __graft_entry__.build()
    import structured_sparse_fp8_b200 as sp
    lib = sp._lib.load()
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    # the streamed kernel on the static scratch (twice), then a decode-sized X
    # (the one-cluster quantiser, no scratch)
    for call, (shape, seed, scale) in enumerate([((64, 4096), 11, 1.0), ((37, 14336), 12, 0.02),
                                                 ((8, 4096), 13, 1.0)]):
        bits = WL.random_bits(shape, seed, scale=scale)
        x = _dev_bf16(bits, dev)
        q = torch.empty(shape, dtype=torch.uint8, device=dev)
        s = torch.empty(1, dtype=torch.float32, device=dev)
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        rc = lib.fp8_quantize_pertensor_static(x.data_ptr(), shape[0], shape[1], q.data_ptr(),
                                               s.data_ptr(), st.data_ptr(), stream)
        assert rc == 0, lib.sp24_status_str(rc)
        ref_q, ref_s = sp.fp8_quantize_pertensor(x)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert s.item() == ref_s.item(), f"call {call}: scale differs"
        assert torch.equal(q, ref_q), f"call {call}: codes differ"
        oq, osx = O.quantize_pertensor(bits)
        assert s.item() == float(osx), f"call {call}: scale differs from the oracle"
        assert np.array_equal(q.cpu().numpy(), oq), f"call {call}: codes differ from the oracle"
