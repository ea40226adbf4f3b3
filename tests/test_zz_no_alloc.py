"""The no-allocation decode-attention entry point, called through the C ABI.

Some callers cannot allocate device memory for a workspace (an engine that
gave all free device memory to its KV-page pool, or a C host program with no
device allocator). dualflow_decode_attn_noalloc serves them from a fixed
scratch array inside the library. This file is collected last on purpose:
if it fails, a run that stops at the first failure has already run every
other test. It passes alone in a fresh process and after the other tests.
"""

import ctypes

import pytest
import torch

from dual_flow_transformer_b200 import _lib as L
from dual_flow_transformer_b200 import api, synth
from tests.helpers import assert_close, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(lib, d, B, Hq, Hkv, D, max_len, o1, o2, num_splits=0, err=None):
    return lib.dualflow_decode_attn_noalloc(
        d["q1"].data_ptr(), d["q2raw"].data_ptr(), d["a"].data_ptr(), d["q1"].stride(0),
        d["k_cache"].data_ptr(), d["v_cache"].data_ptr(), d["block_table"].data_ptr(),
        d["block_table"].shape[1], d["seqlens"].data_ptr(), max_len, o1.data_ptr(), o2.data_ptr(),
        o1.stride(0), B, Hq, Hkv, D, 64, d["k_cache"].shape[0], 0.0, L.DF_BF16, num_splits,
        None if err is None else err.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_the_workspace_entry_point_on_two_calls_in_a_row(cuda_device):
    lib = L.load()
    import dataclasses
    w = dataclasses.replace(synth.WORKLOADS["gqa"], B=4, Hq=8, Hkv=2, len_lo=900, len_hi=3000,
                            seed=77)
    inp = synth.make_attn_inputs(w)
    d = to_dev(inp, cuda_device)
    max_len = int(inp["seqlens"].max())
    assert api.decode_attn_num_splits(w.B, w.Hkv, max_len) > 1  # the scratch is really used
    need = api.decode_attn_workspace_size(w.B, w.Hq, w.Hkv, w.D, max_len)
    assert 0 < need <= L.DF_DECODE_ATTN_NOALLOC_SCRATCH_BYTES
    r1, r2 = api.decode_attn(d["q1"], d["q2raw"], d["a"], d["k_cache"], d["v_cache"],
                             d["block_table"], d["seqlens"], max_len)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    for call in range(2):
        o1 = torch.full_like(d["q1"], float("nan"))
        o2 = torch.full_like(d["q1"], float("nan"))
        st = _noalloc(lib, d, w.B, w.Hq, w.Hkv, w.D, max_len, o1, o2, err=err)
        torch.cuda.synchronize()
        assert st == L.DF_OK, L.status_string(st)
        assert int(err.item()) == 0
        assert_close(o1.cpu(), r1.cpu().double().numpy(), "bf16", "noalloc o1, call %d" % call)
        assert_close(o2.cpu(), r2.cpu().double().numpy(), "bf16", "noalloc o2, call %d" % call)


def test_noalloc_rejects_requests_beyond_its_scratch(cuda_device):
    lib = L.load()
    B, Hq, Hkv, D, max_len, splits = 64, 32, 8, 128, 131072, 64
    assert api.decode_attn_workspace_size(B, Hq, Hkv, D, max_len, splits) > \
        L.DF_DECODE_ATTN_NOALLOC_SCRATCH_BYTES
    fake = 0x7f0000000000  # never dereferenced: the size check comes first
    st = lib.dualflow_decode_attn_noalloc(fake, fake, fake, 0, fake, fake, fake, 2048, fake,
                                          max_len, fake, fake, 0, B, Hq, Hkv, D, 64, 4096, 0.0,
                                          L.DF_BF16, splits, None, None)
    assert st == L.DF_ERR_WORKSPACE
