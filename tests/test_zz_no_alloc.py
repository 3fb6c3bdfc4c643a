"""The allocation-free quantize entry point (qlora_nf4_quantize_noalloc),
called through the C ABI, gives exactly what qlora_nf4_quantize gives with a
caller-allocated workspace, on two calls in a row with different weights (so
that anything left in its shared scratch from the first call would show).

Kept in its own file, collected last, so a run that stops at the first
failure has already run every other test.
"""
import ctypes as C

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dq,codebook", [(True, "nf4"), (False, "nf4"), (False, "int4")])
def test_noalloc_quantize_matches_workspace_entry_point(dq, codebook):
    import bit_nf4_quantized_pack_b200 as q
    from bit_nf4_quantized_pack_b200 import _lib
    dev = torch.device("cuda", 0)
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, (K, N, seed) in enumerate([(1024, 4160, 1), (2048, 3008, 2)]):
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        W = (torch.randn((K, N), generator=g, device=dev) * 0.02).to(torch.bfloat16)
        W[3, :64] = 0.0                                  # an all-zero block
        ref = q.quantize(W, double_quant=dq, codebook=codebook)   # workspace entry point
        out = q.NF4Weight.empty((K, N), dq, dev, codebook=1 if codebook == "int4" else 0)
        st = out.cstruct()
        status = q.new_status(dev)
        rc = _lib.lib.qlora_nf4_quantize_noalloc(C.c_void_p(W.data_ptr()), _lib.QLORA_DTYPE_BF16,
                                                C.byref(st), C.c_void_p(status.data_ptr()), stream)
        assert rc == _lib.QLORA_OK, (call, rc)
        code, mask = q.status_sync(status)
        assert code == 0, (call, mask)
        assert torch.equal(out.packed, ref.packed), call
        if dq:
            assert torch.equal(out.code8, ref.code8), call
            assert torch.equal(out.s2.view(torch.int32), ref.s2.view(torch.int32)), call
            assert torch.equal(out.offset.view(torch.int32), ref.offset.view(torch.int32)), call
        else:
            assert torch.equal(out.absmax.view(torch.int32), ref.absmax.view(torch.int32)), call


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from bit_nf4_quantized_pack_b200 import _lib
    st = _lib.NF4StateC()
    st.numel, st.blocksize, st.double_quant, st.dq_blocksize, st.codebook = \
        _lib.NOALLOC_MAX_NUMEL + 2, 64, 1, 256, 0
    st.packed = st.code8 = st.s2 = st.offset = 4096
    rc = _lib.lib.qlora_nf4_quantize_noalloc(C.c_void_p(4096), 0, C.byref(st), None, None)
    assert rc == _lib.QLORA_ERR_UNSUPPORTED
