"""Failure detection on the GPU without a fault.

A wait that nothing completes runs out after its limit, the kernel raises
QLORA_ERR_TIMEOUT in the status word and returns; the host reads the status
and the context keeps working (a quantization right after it is bit-exact).
Bad inputs are reported the same way (non-finite weights) or rejected on the
host before any launch (null pointers, short workspace: tests/test_abi.py).
"""
import ctypes as C
import time

import numpy as np
import pytest
import torch

from inputs import synthetic as S
from tests._gpu_util import to_dev

pytestmark = pytest.mark.gpu


def _q():
    import bit_nf4_quantized_pack_b200 as q
    return q


def test_bounded_wait_times_out_and_context_survives():
    from oracle import nf4
    q = _q()
    st = q.new_status()
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    t0 = time.perf_counter()
    rc = q.lib.qlora_selftest_bounded_wait(50_000_000, C.c_void_p(st.data_ptr()), stream)
    assert rc == 0
    code, mask = q.status_sync(st)
    dt = time.perf_counter() - t0
    assert code == 6 and mask == 1 << 6, (code, mask)      # QLORA_ERR_TIMEOUT
    assert 0.04 <= dt < 5.0
    # the context is intact: quantize right after, bit-exact against the oracle
    q.status_clear(st)
    w = S.normal(5, 0, 0, (64, 128), 0.02)
    w = S.f32_to_bf16_values(w)
    wq = q.quantize(to_dev(w), double_quant=False, status=st)
    assert q.status_sync(st) == (0, 0)
    codes, absmax = nf4.quantize_nf4(w.ravel())
    payload, _ = nf4.pack_codes(codes)
    assert np.array_equal(wq.packed.cpu().numpy(), payload)

