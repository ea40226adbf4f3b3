"""Host-only checks of the C ABI: the library loads without a GPU, exports every
symbol the header declares, and rejects invalid arguments with the documented
status BEFORE touching the device (no test here can launch a kernel: every
call below carries at least one invalid argument)."""

import ctypes
import os
import re

import pytest

from dual_flow_transformer_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dualflow.h")

FAKE = 0x7f0000000000  # 4 KiB-aligned fake device address (never dereferenced)


def declared_symbols():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dualflow_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    return L.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
        assert n in L.SIGNATURES, "binding lacks a signature for " + n


def test_version_and_status_strings(lib):
    assert lib.dualflow_abi_version() == 1
    for s in range(7):
        assert lib.dualflow_status_string(s).decode().startswith("DF_")
    assert lib.dualflow_status_string(99)


def _attn(lib, **over):
    a = dict(q1=FAKE, q2raw=FAKE, a=FAKE, qs=0, kc=FAKE, vc=FAKE, tbl=FAKE, mbps=4, sl=FAKE,
             maxlen=200, o1=FAKE, o2=FAKE, os=0, B=2, Hq=8, Hkv=2, D=128, bs=64, nb=8,
             scale=0.0, dtype=L.DF_BF16, ns=0, ws=FAKE, wsb=1 << 30, err=None, stream=None)
    a.update(over)
    return lib.dualflow_decode_attn(a["q1"], a["q2raw"], a["a"], a["qs"], a["kc"], a["vc"], a["tbl"],
                                    a["mbps"], a["sl"], a["maxlen"], a["o1"], a["o2"], a["os"],
                                    a["B"], a["Hq"], a["Hkv"], a["D"], a["bs"], a["nb"], a["scale"],
                                    a["dtype"], a["ns"], a["ws"], a["wsb"], a["err"], a["stream"])


@pytest.mark.parametrize("over,status", [
    (dict(q1=None), L.DF_ERR_NULL),
    (dict(kc=None), L.DF_ERR_NULL),
    (dict(tbl=None), L.DF_ERR_NULL),
    (dict(o1=None, o2=None), L.DF_ERR_NULL),
    (dict(o1=None, q2raw=None), L.DF_ERR_NULL),
    (dict(Hq=6, Hkv=4), L.DF_ERR_SHAPE),
    (dict(B=0), L.DF_ERR_SHAPE),
    (dict(maxlen=0), L.DF_ERR_SHAPE),
    (dict(maxlen=257), L.DF_ERR_SHAPE),          # above max_blocks_per_seq * 64
    (dict(qs=100), L.DF_ERR_SHAPE),              # smaller than Hq * D
    (dict(ns=-1), L.DF_ERR_SHAPE),
    (dict(D=96), L.DF_ERR_UNSUPPORTED),
    (dict(bs=32, maxlen=100), L.DF_ERR_UNSUPPORTED),
    (dict(Hq=16, Hkv=2), L.DF_ERR_UNSUPPORTED),  # 8 query rows per KV head and flow
    (dict(dtype=7), L.DF_ERR_UNSUPPORTED),
    (dict(q1=FAKE + 2), L.DF_ERR_ALIGN),
    (dict(kc=FAKE + 8), L.DF_ERR_ALIGN),
    (dict(qs=1025), L.DF_ERR_ALIGN),
    (dict(ws=None, ns=4), L.DF_ERR_WORKSPACE),
    (dict(wsb=16, ns=4), L.DF_ERR_WORKSPACE),
    (dict(ws=FAKE + 16, ns=4), L.DF_ERR_WORKSPACE),
])
def test_decode_attn_rejects_invalid_arguments(lib, over, status):
    assert _attn(lib, **over) == status


def test_decode_attn_plan(lib):
    ns = lib.dualflow_decode_attn_num_splits
    ws = lib.dualflow_decode_attn_workspace_size
    assert ns(1, 2, 129, 64, 0) >= 1
    assert ns(1, 1, 64, 64, 5) == 1                # never more splits than pages
    assert ns(64, 8, 4097, 64, 3) == 3
    for B, Hkv, L_ in [(32, 32, 2048), (64, 8, 8192), (8, 8, 131072), (64, 8, 4097), (1, 2, 129)]:
        s = ns(B, Hkv, L_, 64, 0)
        pages = -(-L_ // 64)
        chunk = -(-pages // s)
        assert 1 <= s <= pages and -(-pages // chunk) == s
        if s > 1:
            # arrival counters + partials (o and (max, sum)) of every split
            assert ws(B, 2 * Hkv, Hkv, 128, L_, 64, 0) >= B * Hkv * 4 + B * 2 * 2 * Hkv * s * 130 * 4
        else:
            assert ws(B, 2 * Hkv, Hkv, 128, L_, 64, 0) == 0
    assert ns(0, 1, 10, 64, 0) == 0 and ws(0, 1, 1, 64, 10, 64, 0) == 0
    nl = lib.dualflow_decode_attn_num_launches
    assert nl(8, 8, 131072, 64, 0, L.DF_BF16) == 1  # the combine runs inside the kernel
    assert nl(8, 8, 131072, 64, 0, L.DF_FP32) == 2 and nl(1, 2, 129, 64, 1, L.DF_FP32) == 1
    # automatic plan: one CTA per (sequence, KV head) unit once the units fill
    # the 296 resident slots (2 per SM); otherwise ~2 waves, chunks >= 8 pages
    assert ns(64, 8, 4097, 64, 0) == 1 and ns(32, 32, 2048, 64, 0) == 1
    assert ns(8, 8, 131072, 64, 0) == 10           # ceil(592 / 64) splits
    assert ns(4, 2, 4096, 64, 0) == 8               # capped: 64 pages / 8
    assert nl(0, 8, 4097, 64, 0, L.DF_BF16) == 0 and nl(1, 1, 64, 64, 0, 9) == 0


def _append(lib, **over):
    a = dict(kn=FAKE, vn=FAKE, st=0, kc=FAKE, vc=FAKE, tbl=FAKE, mbps=4, pos=FAKE, B=2, Hkv=2,
             D=128, bs=64, nb=8, dtype=L.DF_BF16, err=None, stream=None)
    a.update(over)
    return lib.dualflow_kv_append(a["kn"], a["vn"], a["st"], a["kc"], a["vc"], a["tbl"], a["mbps"],
                                  a["pos"], a["B"], a["Hkv"], a["D"], a["bs"], a["nb"], a["dtype"],
                                  a["err"], a["stream"])


@pytest.mark.parametrize("over,status", [
    (dict(kn=None), L.DF_ERR_NULL),
    (dict(pos=None), L.DF_ERR_NULL),
    (dict(B=0), L.DF_ERR_SHAPE),
    (dict(st=10), L.DF_ERR_SHAPE),
    (dict(dtype=5), L.DF_ERR_UNSUPPORTED),
    (dict(D=4), L.DF_ERR_ALIGN),               # 8-byte rows cannot use 16-byte copies
    (dict(kc=FAKE + 4), L.DF_ERR_ALIGN),
])
def test_kv_append_rejects_invalid_arguments(lib, over, status):
    assert _append(lib, **over) == status


def test_rmsnorm_rejects_invalid_arguments(lib):
    f = lib.dualflow_rmsnorm
    assert f(None, 0, None, FAKE, 0, 4, 64, 1e-5, None) == L.DF_ERR_NULL
    assert f(FAKE, 0, None, FAKE, 0, 0, 64, 1e-5, None) == L.DF_ERR_SHAPE
    assert f(FAKE, 0, None, FAKE, 0, 4, 60, 1e-5, None) == L.DF_ERR_UNSUPPORTED
    assert f(FAKE + 2, 0, None, FAKE, 0, 4, 64, 1e-5, None) == L.DF_ERR_ALIGN
    assert f(FAKE, 0, None, FAKE, 0, 4, 64, -1.0, None) == L.DF_ERR_SHAPE


def test_grouped_proj_chain_rejects_invalid_next_projection(lib):
    f = lib.dualflow_grouped_proj_chain
    base = [FAKE, 0, 64, 64, FAKE, 4096, 4096, 4096, FAKE, 0, 0, None, None, 0, FAKE, 1 << 30]
    tail = [None, None]
    assert f(*base, FAKE, 4000, 4096, 0, *tail) == L.DF_ERR_UNSUPPORTED   # N_next % 128
    assert f(*base, FAKE, 4096, 4000, 0, *tail) == L.DF_ERR_UNSUPPORTED   # K_next % 64
    assert f(*base, FAKE, 4096, 4096, 7, *tail) == L.DF_ERR_UNSUPPORTED   # epilogue_next
    assert f(*base, FAKE + 8, 4096, 4096, 0, *tail) == L.DF_ERR_ALIGN     # w_next alignment
    assert f(None, *base[1:], FAKE, 4096, 4096, 0, *tail) == L.DF_ERR_NULL


def test_mixture_head_rejects_invalid_arguments(lib):
    f = lib.dualflow_mixture_head
    ok = dict(lg=FAKE, ld=0, B=4, V=4096, dt=L.DF_BF16, p=FAKE, ldp=0, a=FAKE, st=None)

    def call(**over):
        a = dict(ok)
        a.update(over)
        return f(a["lg"], a["ld"], a["B"], a["V"], a["dt"], a["p"], a["ldp"], a["a"], a["st"])

    assert call(lg=None) == L.DF_ERR_NULL
    assert call(p=None) == L.DF_ERR_NULL
    assert call(B=0) == L.DF_ERR_SHAPE
    assert call(ld=100) == L.DF_ERR_SHAPE          # row stride below V
    assert call(V=4100) == L.DF_ERR_UNSUPPORTED    # V % 8
    assert call(dt=7) == L.DF_ERR_UNSUPPORTED
    assert call(lg=FAKE + 8) == L.DF_ERR_ALIGN
    assert call(ldp=4098) == L.DF_ERR_ALIGN
    assert call(ld=4100) == L.DF_ERR_ALIGN
    sl = lib.dualflow_mixture_head_slices
    assert sl(64, 32000) == 8 and sl(1, 32000) == 8 and sl(4, 1024) == 1 and sl(0, 8) == 0


def test_moe_entry_points_reject_invalid_arguments(lib):
    r = lib.dualflow_moe_route
    assert r(None, 0, 4, 256, FAKE, 8, 2, 2, FAKE, FAKE, FAKE, None, None) == L.DF_ERR_NULL
    assert r(FAKE, 0, 65, 256, FAKE, 8, 2, 2, FAKE, FAKE, FAKE, None, None) == L.DF_ERR_UNSUPPORTED
    assert r(FAKE, 0, 4, 256, FAKE, 8, 3, 2, FAKE, FAKE, FAKE, None, None) == L.DF_ERR_SHAPE
    assert r(FAKE, 0, 4, 256, FAKE, 8, 2, 9, FAKE, FAKE, FAKE, None, None) == L.DF_ERR_UNSUPPORTED
    assert r(FAKE, 0, 4, 252, FAKE, 8, 2, 2, FAKE, FAKE, FAKE, None, None) == L.DF_ERR_UNSUPPORTED
    assert r(FAKE + 8, 0, 4, 256, FAKE, 8, 2, 2, FAKE, FAKE, FAKE, None, None) == L.DF_ERR_ALIGN
    dsp = lib.dualflow_moe_dispatch
    assert dsp(FAKE, 0, 4, 256, FAKE, 8, 2, 2, None, FAKE, FAKE, None, None, None) == L.DF_ERR_NULL
    assert dsp(FAKE, 0, 0, 256, FAKE, 8, 2, 2, FAKE, FAKE, FAKE, None, None, None) == L.DF_ERR_SHAPE
    assert dsp(FAKE, 100, 4, 256, FAKE, 8, 2, 2, FAKE, FAKE, FAKE, None, None, None) == L.DF_ERR_SHAPE
    c = lib.dualflow_moe_combine
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 256, 8, 2, 2, None, 0, FAKE, 0, None, None]
    bad = list(args)
    bad[13] = None
    assert c(*bad) == L.DF_ERR_NULL
    bad = list(args)
    bad[14] = 100
    assert c(*bad) == L.DF_ERR_SHAPE
    bad = list(args)
    bad[13] = FAKE + 8
    assert c(*bad) == L.DF_ERR_ALIGN


def test_grouped_proj_batched_rejects_invalid_arguments(lib):
    f = lib.dualflow_grouped_proj_batched
    ok = [FAKE, 0, 0, 64, 64, FAKE, 1024, 512, 0, FAKE, 0, 0, 4, 0, FAKE, 1 << 30,
          None, 0, 0, 0, 1, 0, None, None]

    def call(**over):
        a = list(ok)
        for i, v in over.items():
            a[int(i[1:])] = v
        return f(*a)

    assert call(a0=None) == L.DF_ERR_NULL
    assert call(a12=0) == L.DF_ERR_SHAPE                    # batch
    assert call(a13=2) == L.DF_ERR_UNSUPPORTED              # residual epilogue
    assert call(a2=100) == L.DF_ERR_SHAPE                   # x batch stride below M * K
    assert call(a8=1024 * 512 + 4) == L.DF_ERR_ALIGN        # w batch stride not 16-byte
    nl = lib.dualflow_grouped_proj_batched_num_launches
    assert nl(128, 1024, 512, 2, 4) == 0 and nl(0, 1024, 512, 0, 4) == 0


def _prefill(lib, **over):
    a = dict(q1=FAKE, qs=0, kn=FAKE, vn=FAKE, kvs=0, q2=FAKE, av=FAKE, kc=FAKE, vc=FAKE,
             tbl=FAKE, mbps=8, cu=FAKE, ctx=None, mql=256, msl=400, o1=FAKE, os=0, o2=FAKE,
             B=2, T=300, Hq=8, Hkv=2, D=128, bs=64, nb=16, scale=0.0, dtype=L.DF_BF16,
             ws=FAKE, wsb=1 << 30, err=None, stream=None)
    a.update(over)
    return lib.dualflow_prefill(a["q1"], a["qs"], a["kn"], a["vn"], a["kvs"], a["q2"], a["av"],
                                a["kc"], a["vc"], a["tbl"], a["mbps"], a["cu"], a["ctx"],
                                a["mql"], a["msl"], a["o1"], a["os"], a["o2"], a["B"], a["T"],
                                a["Hq"], a["Hkv"], a["D"], a["bs"], a["nb"], a["scale"],
                                a["dtype"], a["ws"], a["wsb"], a["err"], a["stream"])


@pytest.mark.parametrize("over,status", [
    (dict(q1=None), L.DF_ERR_NULL),
    (dict(o1=None), L.DF_ERR_NULL),
    (dict(cu=None), L.DF_ERR_NULL),
    (dict(vn=None), L.DF_ERR_NULL),               # k_new without v_new
    (dict(T=1), L.DF_ERR_SHAPE),                  # fewer tokens than sequences
    (dict(mql=301), L.DF_ERR_SHAPE),              # chunk bound above T
    (dict(msl=100), L.DF_ERR_SHAPE),              # max_seqlen below max_q_len
    (dict(msl=600), L.DF_ERR_SHAPE),              # beyond the block table
    (dict(Hq=7), L.DF_ERR_SHAPE),
    (dict(qs=8), L.DF_ERR_SHAPE),                 # token stride below Hq * D
    (dict(dtype=L.DF_FP32), L.DF_ERR_UNSUPPORTED),
    (dict(D=96), L.DF_ERR_UNSUPPORTED),
    (dict(bs=32, msl=256), L.DF_ERR_UNSUPPORTED),
    (dict(Hq=16, Hkv=2), L.DF_ERR_UNSUPPORTED),   # auxiliary step needs Hq/Hkv <= 4
    (dict(q1=FAKE + 8), L.DF_ERR_ALIGN),
    (dict(qs=8 * 128 + 4), L.DF_ERR_ALIGN),
    (dict(kn=FAKE + 4), L.DF_ERR_ALIGN),
    (dict(ws=None), L.DF_ERR_WORKSPACE),
    (dict(wsb=16), L.DF_ERR_WORKSPACE),
    (dict(ws=FAKE + 64), L.DF_ERR_WORKSPACE),
])
def test_prefill_rejects_invalid_arguments(lib, over, status):
    assert _prefill(lib, **over) == status


def test_prefill_sizes(lib):
    assert lib.dualflow_prefill_num_launches(1, 1) == 4
    assert lib.dualflow_prefill_num_launches(0, 1) == 3
    assert lib.dualflow_prefill_num_launches(1, 0) == 2
    assert lib.dualflow_prefill_workspace_size(2, 8, 2, 128, 400, 64) > 0
    assert lib.dualflow_prefill_workspace_size(2, 8, 2, 128, 400, 32) == 0


def test_prefill_kernel_choice_is_checked(lib):
    def ex(kernel, D=128, T=300, o1=FAKE):
        return lib.dualflow_prefill_ex(FAKE, 0, FAKE, FAKE, 0, None, None, FAKE, FAKE, FAKE, 8,
                                       FAKE, None, 256, 400, o1, 0, None, 2, T, 8, 2, D, 64, 16,
                                       0.0, L.DF_BF16, kernel, None, 0, None, None)
    assert ex(7) == L.DF_ERR_SHAPE
    assert ex(L.DF_PREFILL_KERNEL_TCGEN05, T=100, o1=FAKE) == L.DF_ERR_SHAPE  # max_q_len > T
    assert ex(L.DF_PREFILL_KERNEL_TCGEN05, o1=FAKE + 4) == L.DF_ERR_UNSUPPORTED
    assert lib.dualflow_prefill_kernel(128, 300, FAKE, 0, 8) == L.DF_PREFILL_KERNEL_TCGEN05
    assert lib.dualflow_prefill_kernel(128, 100, FAKE, 0, 8) == L.DF_PREFILL_KERNEL_MMA_SYNC
    assert lib.dualflow_prefill_kernel(64, 300, FAKE, 0, 8) == L.DF_PREFILL_KERNEL_TCGEN05
    assert lib.dualflow_prefill_kernel(64, 100, FAKE, 0, 8) == L.DF_PREFILL_KERNEL_MMA_SYNC
    assert lib.dualflow_prefill_kernel(96, 300, FAKE, 0, 8) == L.DF_PREFILL_KERNEL_MMA_SYNC
    assert lib.dualflow_prefill_kernel(128, 300, FAKE + 4, 0, 8) == L.DF_PREFILL_KERNEL_MMA_SYNC


def test_selftest_and_split_pre_entries_reject_invalid_arguments(lib):
    # every check below returns before any CUDA call
    assert lib.dualflow_selftest_wait_timeout(None, None) == L.DF_ERR_NULL
    buf = 4096
    assert lib.dualflow_layer_qkv_partials(None, buf, 8, 512, 4, 2, 128, buf, buf, None,
                                           None) == L.DF_ERR_NULL
    assert lib.dualflow_layer_qkv_partials(buf, buf, 0, 512, 4, 2, 128, buf, buf, None,
                                           None) == L.DF_ERR_SHAPE

    def attn(**kw):
        a = dict(part=buf, ss=buf, parts=4, m=8, d=512, eps=1e-5)
        a.update(kw)
        return lib.dualflow_decode_attn_qkv_partials(
            a["part"], a["ss"], a["parts"], a["m"], a["d"], a["eps"], None, buf, buf, buf, 4,
            buf, 200, buf, buf, 0, 4, 2, 128, 64, 100, 0.0, 0, None, 0, None, None)

    assert attn(part=None) == L.DF_ERR_NULL
    assert attn(ss=None) == L.DF_ERR_NULL
    assert attn(parts=0) == L.DF_ERR_SHAPE
    assert attn(parts=5) == L.DF_ERR_SHAPE
    assert attn(m=0) == L.DF_ERR_SHAPE
    assert attn(eps=-1.0) == L.DF_ERR_SHAPE
    assert attn(part=buf + 4) == L.DF_ERR_ALIGN


def test_post_attention_qkv_entry_rejects_invalid_arguments(lib):
    """The layer-stack entry's own checks (before the post-attention launch's
    and before any CUDA call): the next layer's W_qkv is required, and the
    head layout must match the attention width."""
    buf = 4096

    def call(w_qkv=buf, Hq=4, Hkv=2, D=128, q_dim=512):
        return lib.dualflow_layer_post_attention_qkv(
            buf, buf, buf, buf, buf, None, None, 8, 512, q_dim, 1024, 1e-5, buf, buf, buf, buf,
            1 << 20, w_qkv, Hq, Hkv, D, buf, buf, None, None)

    assert call(w_qkv=None) == L.DF_ERR_NULL
    assert call(Hq=0) == L.DF_ERR_SHAPE
    assert call(Hkv=3) == L.DF_ERR_SHAPE        # Hq % Hkv != 0
    assert call(q_dim=256) == L.DF_ERR_SHAPE    # q_dim != Hq * D
    assert call(D=0) == L.DF_ERR_SHAPE
