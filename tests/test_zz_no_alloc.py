"""The no-allocation decode-attention entry point, called through the C ABI.

Some callers cannot allocate device memory for a workspace (an engine that
gave all free device memory to its KV-page pool, or a C host program with no
device allocator). dualflow_decode_attn_noalloc serves them from a fixed
scratch array inside the library. It runs the same plan and the same kernel
as dualflow_decode_attn, so its outputs must be bit-identical to that entry
point's, and within the stated tolerance of the oracle.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test. It passes alone in a fresh
process and after the other tests.
"""

import dataclasses

import pytest
import torch

from dual_flow_transformer_b200 import _lib as L
from dual_flow_transformer_b200 import api, synth
from tests.helpers import assert_attn_close, oracle_attn, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(lib, d, w, max_len, o1, o2, num_splits=0, err=None):
    return lib.dualflow_decode_attn_noalloc(
        d["q1"].data_ptr(), d["q2raw"].data_ptr(), d["a"].data_ptr(), d["q1"].stride(0),
        d["k_cache"].data_ptr(), d["v_cache"].data_ptr(), d["block_table"].data_ptr(),
        d["block_table"].shape[1], d["seqlens"].data_ptr(), max_len, o1.data_ptr(),
        o2.data_ptr(), o1.stride(0), w.B, w.Hq, w.Hkv, w.D, 64, d["k_cache"].shape[0], 0.0,
        L.DF_BF16 if w.dtype == "bf16" else L.DF_FP32, num_splits,
        None if err is None else err.data_ptr(), torch.cuda.current_stream().cuda_stream)


# (name, workload, num_splits): bf16 split in the kernel (arrival counters in
# the scratch), bf16 unsplit (no scratch at all), fp32 split (partials plus a
# separate combine launch, no counters).
CASES = [
    ("bf16-auto", dataclasses.replace(synth.WORKLOADS["gqa"], B=4, Hq=8, Hkv=2, len_lo=900,
                                      len_hi=3000, seed=77), 0),
    ("bf16-one-split", dataclasses.replace(synth.WORKLOADS["gqa"], B=4, Hq=8, Hkv=2,
                                           len_lo=100, len_hi=700, seed=78), 1),
    ("fp32-split", dataclasses.replace(synth.WORKLOADS["tiny"], B=2, Hq=4, Hkv=2, len_lo=300,
                                       len_hi=700, append=False, seed=79), 3),
]


@pytest.mark.parametrize("name,w,num_splits", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_the_workspace_entry_point_on_two_calls_in_a_row(cuda_device, name, w,
                                                                        num_splits):
    lib = L.load()
    inp = synth.make_attn_inputs(w)
    d = to_dev(inp, cuda_device)
    max_len = int(inp["seqlens"].max())
    splits = api.decode_attn_num_splits(w.B, w.Hkv, max_len, num_splits)
    need = api.decode_attn_workspace_size(w.B, w.Hq, w.Hkv, w.D, max_len, num_splits)
    if num_splits == 1:
        assert splits == 1 and need == 0  # no scratch is used at all
    else:
        assert splits > 1 and 0 < need <= L.DF_DECODE_ATTN_NOALLOC_SCRATCH_BYTES
    # the workspace entry point first, on the same stream, then the no-alloc one
    r1, r2 = api.decode_attn(d["q1"], d["q2raw"], d["a"], d["k_cache"], d["v_cache"],
                             d["block_table"], d["seqlens"], max_len, num_splits=num_splits)
    torch.cuda.synchronize()
    ref1, ref2 = oracle_attn(inp)
    dt = "bf16" if w.dtype == "bf16" else "fp32"
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    for call in range(2):
        o1 = torch.full_like(d["q1"], float("nan"))
        o2 = torch.full_like(d["q1"], float("nan"))
        st = _noalloc(lib, d, w, max_len, o1, o2, num_splits=num_splits, err=err)
        torch.cuda.synchronize()
        assert st == L.DF_OK, L.status_string(st)
        assert int(err.item()) == 0
        # same plan, same kernel: bit for bit the workspace entry point's result
        assert torch.equal(o1.view(torch.int16 if dt == "bf16" else torch.int32),
                           r1.view(torch.int16 if dt == "bf16" else torch.int32)), (name, call)
        assert torch.equal(o2.view(torch.int16 if dt == "bf16" else torch.int32),
                           r2.view(torch.int16 if dt == "bf16" else torch.int32)), (name, call)
        assert_attn_close(o1.cpu(), ref1, dt, "%s noalloc o1, call %d" % (name, call))
        assert_attn_close(o2.cpu(), ref2, dt, "%s noalloc o2, call %d" % (name, call))


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


def test_noalloc_rejected_call_leaves_the_scratch_alone(cuda_device):
    # A call that fails an argument check (here a misaligned cache pointer)
    # returns before any device work: a later valid call still matches.
    lib = L.load()
    w = CASES[0][1]
    inp = synth.make_attn_inputs(w)
    d = to_dev(inp, cuda_device)
    max_len = int(inp["seqlens"].max())
    o1 = torch.empty_like(d["q1"])
    o2 = torch.empty_like(d["q1"])
    class Shifted:  # the cache pointer moved by 2 bytes: not 16-byte aligned
        shape = d["k_cache"].shape

        @staticmethod
        def data_ptr():
            return d["k_cache"].data_ptr() + 2

    bad = dict(d, k_cache=Shifted())
    st = _noalloc(lib, bad, w, max_len, o1, o2)
    assert st == L.DF_ERR_ALIGN
    st = _noalloc(lib, d, w, max_len, o1, o2)
    torch.cuda.synchronize()
    assert st == L.DF_OK
    ref1, ref2 = oracle_attn(inp)
    assert_attn_close(o1.cpu(), ref1, "bf16", "noalloc o1 after a rejected call")
    assert_attn_close(o2.cpu(), ref2, "bf16", "noalloc o2 after a rejected call")
