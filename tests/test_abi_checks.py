"""Host-side argument checks of the C ABI: every malformed call returns its
status before anything is launched (dsa_launch_counter unchanged).

The calls carry fake device addresses that nothing dereferences, so this
module runs only on a host without a CUDA device: there, a call that passes
every host check stops at the device lookup with DSA_ERR_CUDA. That is the
control below -- the unmodified arguments reach the device lookup -- and each
case changes one field of them and must get its own status instead."""
import ctypes
import os

import pytest
import torch

pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="fake device pointers: host-only checks")

FAKE = 0x7F0000000000          # 16-byte (and 256-byte) aligned, never dereferenced


@pytest.fixture(scope="module")
def dsa():
    from sparse_attention_long_tcgen05_b200 import _build
    _build.build()
    from sparse_attention_long_tcgen05_b200 import dsa
    return dsa


def _contig(dsa, n=1):
    return dsa.KvLayout(dsa.DSA_KV_CONTIGUOUS, 0, None, 0, 0, 0, None)


def _paged(dsa):
    return dsa.KvLayout(dsa.DSA_KV_PAGED, 64, FAKE + 0x1000, 2048, 2048, 4096, FAKE + 0x2000,
                        None, None, 0)


def _indexer(dsa, kv=None, n_q=4096, n_keys=4096):
    kv = kv if kv is not None else _contig(dsa)
    return dsa.IndexerIn(dsa.DSA_E4M3, n_q, n_keys, 64, 128, FAKE + 0x10000, 8192,
                         FAKE + 0x20000, FAKE + 0x30000, 128, FAKE + 0x40000, FAKE + 0x50000,
                         64, kv)


def _attn(dsa, kv=None, n_q=4096, n_keys=4096):
    kv = kv if kv is not None else _contig(dsa)
    return dsa.AttnIn(dsa.DSA_BF16, n_q, n_keys, 128, 576, 512, 576 ** -0.5,
                      FAKE + 0x60000, 128 * 576, FAKE + 0x70000, 576, None, 0, kv)


def _mut(s, **kw):
    c = type(s)()
    ctypes.memmove(ctypes.byref(c), ctypes.byref(s), ctypes.sizeof(s))
    s = c
    for k, v in kw.items():
        setattr(s, k, v)
    return s


def _p(x):
    return ctypes.c_void_p(x) if x is not None else None


def _scores(dsa, ind, rows=None, n_rows=4, scores=FAKE + 0x80000, ld=4096, n_cols=4096):
    return dsa.LIB.dsa_indexer_scores(ctypes.byref(ind), _p(rows), n_rows, _p(scores), ld,
                                      n_cols, None, 0, None)


def _topk(dsa, scores=FAKE, ld=4096, pos=FAKE + 0x1000, n_rows=4, k=2048, idx=FAKE + 0x2000,
          ld_idx=2048):
    return dsa.LIB.dsa_topk(_p(scores), ld, _p(pos), n_rows, k, _p(idx), ld_idx, None)


def _mqa(dsa, att, idx=FAKE + 0x1000, ld_idx=2048, k=2048, out=FAKE + 0x2000):
    return dsa.LIB.dsa_sparse_mqa_fwd(ctypes.byref(att), _p(idx), ld_idx, k, _p(out), None,
                                      None, 0, None)


def _forward(dsa, ind, att, k=2048, ws=FAKE + 0x100000, ws_bytes=1 << 34, out=FAKE + 0x2000):
    return dsa.LIB.dsa_forward(ctypes.byref(ind), ctypes.byref(att), k, None, _p(out), None,
                               _p(ws), ws_bytes, None)


def _select(dsa, ind, k=2048, idx=FAKE + 0x3000, ld_idx=2048, ws=FAKE + 0x100000,
            ws_bytes=1 << 34):
    return dsa.LIB.dsa_select(ctypes.byref(ind), k, _p(idx), ld_idx, _p(ws), ws_bytes, None)


def _expect(dsa, status, call):
    n0 = dsa.dsa_launch_counter()
    got = call()
    assert dsa.dsa_launch_counter() == n0, "a rejected call launched a kernel"
    assert got == status, (dsa.status_string(got), dsa.status_string(status))


def test_control_calls_pass_every_host_check(dsa):
    """The unmodified arguments reach the device lookup (no device here)."""
    ind, att = _indexer(dsa), _attn(dsa)
    E = dsa.DSA_ERR_CUDA
    _expect(dsa, E, lambda: _scores(dsa, ind))
    _expect(dsa, E, lambda: _topk(dsa))
    _expect(dsa, E, lambda: _mqa(dsa, att))
    _expect(dsa, E, lambda: _forward(dsa, ind, att))
    _expect(dsa, E, lambda: _select(dsa, ind))
    pind, patt = _indexer(dsa, _paged(dsa), 64, 0), _attn(dsa, _paged(dsa), 64, 0)
    _expect(dsa, E, lambda: _forward(dsa, pind, patt))
    _expect(dsa, E, lambda: dsa.LIB.dsa_select_noalloc(ctypes.byref(ind), 2048,
                                                       _p(FAKE), 2048, None))


def test_indexer_argument_checks(dsa):
    ind = _indexer(dsa)
    INV, UNS = dsa.DSA_ERR_INVALID_ARG, dsa.DSA_ERR_UNSUPPORTED
    _expect(dsa, INV, lambda: dsa.LIB.dsa_indexer_scores(None, None, 4, _p(FAKE), 4096, 4096,
                                                         None, 0, None))
    cases = [
        (INV, dict(q=None)), (INV, dict(k=None)), (INV, dict(w=None)),
        (INV, dict(q_scale=None)), (INV, dict(k_scale=None)),
        (INV, dict(q=FAKE + 0x10008)),            # not 16-byte aligned (TMA)
        (INV, dict(k=FAKE + 0x30004)),
        (INV, dict(k_scale=FAKE + 0x40004)),
        (INV, dict(ld_q=8192 + 8)),               # row stride not a multiple of 16 bytes
        (INV, dict(ld_k=136)),
        (INV, dict(ld_k=64)),                     # ld_k < dim
        (INV, dict(ld_w=32)),                     # ld_w < heads
        (INV, dict(n_keys=100)),                  # fewer keys than queries
        (INV, dict(n_q=0)),
        (UNS, dict(heads=32, ld_q=4096)),         # E4M3 path is built for 64 x 128
        (UNS, dict(dim=64)),
        (UNS, dict(dtype=7)),
    ]
    for status, kw in cases:
        bad = _mut(ind, **kw)
        _expect(dsa, status, lambda: _scores(dsa, bad))
    _expect(dsa, INV, lambda: _scores(dsa, ind, scores=None))
    _expect(dsa, INV, lambda: _scores(dsa, ind, n_rows=0))
    _expect(dsa, INV, lambda: _scores(dsa, ind, n_rows=4097))      # more rows than queries
    _expect(dsa, INV, lambda: _scores(dsa, ind, n_cols=0))
    _expect(dsa, INV, lambda: _scores(dsa, ind, ld=100, n_cols=4096))
    # F32 indexer: no scales, contiguous only, bounded dims
    f32 = _mut(ind, dtype=dsa.DSA_F32, heads=4, dim=32, ld_q=128, ld_k=32, ld_w=4,
               q_scale=None, k_scale=None)
    _expect(dsa, dsa.DSA_ERR_CUDA, lambda: _scores(dsa, f32))
    _expect(dsa, INV, lambda: _scores(dsa, _mut(f32, q_scale=FAKE)))
    _expect(dsa, UNS, lambda: _scores(dsa, _mut(f32, dim=30, ld_k=32)))
    _expect(dsa, UNS, lambda: _scores(dsa, _mut(f32, heads=65, ld_q=65 * 32, ld_w=65)))
    _expect(dsa, UNS, lambda: _scores(dsa, _mut(f32, kv=_paged(dsa))))


def test_paged_layout_checks(dsa):
    INV, UNS = dsa.DSA_ERR_INVALID_ARG, dsa.DSA_ERR_UNSUPPORTED
    lay = _paged(dsa)
    ind = _indexer(dsa, lay, 64, 0)
    cases = [
        (UNS, dict(page_size=32)), (INV, dict(block_table=None)), (INV, dict(ctx_lens=None)),
        (INV, dict(max_pages=0)), (INV, dict(num_pages=0)), (INV, dict(ld_block_table=100)),
        (INV, dict(kind=5)), (INV, dict(max_pages=1 << 26, ld_block_table=1 << 26)),
        (INV, dict(n_seq=-1)),
        (INV, dict(n_seq=10)),            # 64 queries, no q_seq: one sequence per query needed
    ]
    for status, kw in cases:
        bad = _mut(ind, kv=_mut(lay, **kw))
        _expect(dsa, status, lambda: _scores(dsa, bad, n_cols=64))
    # a score row may not be wider than the block table covers
    _expect(dsa, INV, lambda: _scores(dsa, ind, n_cols=2048 * 64 + 1, ld=2048 * 64 + 1))


def test_topk_argument_checks(dsa):
    INV = dsa.DSA_ERR_INVALID_ARG
    for kw in (dict(k=0), dict(k=2049), dict(k=-3), dict(ld_idx=100), dict(scores=None),
               dict(pos=None), dict(idx=None), dict(n_rows=0), dict(ld=0)):
        _expect(dsa, INV, lambda: _topk(dsa, **kw))


def test_attention_argument_checks(dsa):
    att = _attn(dsa)
    INV, UNS = dsa.DSA_ERR_INVALID_ARG, dsa.DSA_ERR_UNSUPPORTED
    cases = [
        (INV, dict(q=None)), (INV, dict(kv=None)),
        (INV, dict(scale=0.0)), (INV, dict(scale=float("nan"))), (INV, dict(scale=-1.0)),
        (INV, dict(scale=float("inf"))),
        (INV, dict(q=FAKE + 0x60004)), (INV, dict(kv=FAKE + 0x70002)),
        (INV, dict(ld_q=128 * 576 + 4)),          # bf16 stride not a multiple of 16 bytes
        (INV, dict(ld_kv=580)),
        (INV, dict(ld_kv=512)),                   # ld_kv < d_qk
        (INV, dict(n_keys=10)),
        (UNS, dict(heads=64, ld_q=64 * 576)),     # BF16 path is built for 128 / 576 / 512
        (UNS, dict(d_v=256)),
        (UNS, dict(v=FAKE + 0x90000, ld_v=512)),  # separate V only for F32
        (UNS, dict(dtype=9)),
    ]
    for status, kw in cases:
        bad = _mut(att, **kw)
        _expect(dsa, status, lambda: _mqa(dsa, bad))
    _expect(dsa, INV, lambda: dsa.LIB.dsa_sparse_mqa_fwd(None, _p(FAKE), 2048, 2048, _p(FAKE),
                                                         None, None, 0, None))
    _expect(dsa, INV, lambda: _mqa(dsa, att, idx=None))
    _expect(dsa, INV, lambda: _mqa(dsa, att, out=None))
    _expect(dsa, INV, lambda: _mqa(dsa, att, out=FAKE + 0x2008))
    _expect(dsa, INV, lambda: _mqa(dsa, att, k=0))
    _expect(dsa, INV, lambda: _mqa(dsa, att, k=2049))
    _expect(dsa, INV, lambda: _mqa(dsa, att, ld_idx=1000))


def test_forward_and_select_checks(dsa):
    ind, att = _indexer(dsa), _attn(dsa)
    INV, UNS, WS = dsa.DSA_ERR_INVALID_ARG, dsa.DSA_ERR_UNSUPPORTED, \
        dsa.DSA_ERR_WORKSPACE_TOO_SMALL
    need = dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD, dsa._Keep(ind, []), None, 0, 0, 2048)
    need_sel = dsa.dsa_workspace_size(dsa.DSA_OP_SELECT, dsa._Keep(ind, []), None, 0, 0, 2048)
    _expect(dsa, dsa.DSA_ERR_CUDA, lambda: _forward(dsa, ind, att, ws_bytes=need))
    _expect(dsa, WS, lambda: _forward(dsa, ind, att, ws_bytes=need - 1))
    _expect(dsa, WS, lambda: _forward(dsa, ind, att, ws=None))
    _expect(dsa, WS, lambda: _forward(dsa, ind, att, ws=FAKE + 0x100010))   # not 256-aligned
    _expect(dsa, INV, lambda: _forward(dsa, ind, att, k=0))
    _expect(dsa, INV, lambda: _forward(dsa, ind, att, k=4096))
    _expect(dsa, INV, lambda: _forward(dsa, ind, att, out=None))
    _expect(dsa, INV, lambda: _forward(dsa, ind, _mut(att, n_q=4000)))
    _expect(dsa, INV, lambda: _forward(dsa, ind, _mut(att, n_keys=5000)))
    f32 = _mut(att, dtype=dsa.DSA_F32, heads=8, d_qk=64, d_v=64, ld_q=512, ld_kv=64)
    _expect(dsa, UNS, lambda: _forward(dsa, ind, f32))                       # mixed dtypes
    pind, patt = _indexer(dsa, _paged(dsa), 64, 0), _attn(dsa, _paged(dsa), 64, 0)
    _expect(dsa, INV, lambda: _forward(dsa, pind, att))                      # layouts differ
    for kw in (dict(block_table=FAKE + 0x5000), dict(ctx_lens=FAKE + 0x5000),
               dict(q_pos=FAKE + 0x5000), dict(q_seq=FAKE + 0x5000, n_seq=64),
               dict(max_pages=1024)):
        _expect(dsa, INV, lambda: _forward(dsa, pind, _mut(patt, kv_layout=_mut(
            _paged(dsa), **kw))))
    # several queries per sequence: q_seq / q_pos given, fewer sequences than queries
    mlay = _mut(_paged(dsa), q_seq=FAKE + 0x6000, q_pos=FAKE + 0x7000, n_seq=8)
    _expect(dsa, dsa.DSA_ERR_CUDA, lambda: _forward(dsa, _indexer(dsa, mlay, 64, 0),
                                                    _attn(dsa, mlay, 64, 0)))
    _expect(dsa, dsa.DSA_ERR_CUDA, lambda: _select(dsa, ind, ws_bytes=need_sel))
    _expect(dsa, WS, lambda: _select(dsa, ind, ws_bytes=need_sel - 1))
    _expect(dsa, INV, lambda: _select(dsa, ind, idx=None))
    _expect(dsa, INV, lambda: _select(dsa, ind, ld_idx=2047))


def test_workspace_size_checks(dsa):
    ind = dsa._Keep(_indexer(dsa), [])
    out = ctypes.c_size_t(0)
    INV = dsa.DSA_ERR_INVALID_ARG
    assert dsa.LIB.dsa_workspace_size(dsa.DSA_OP_FORWARD, ctypes.byref(ind.struct), None, 0, 0,
                                      2048, None) == INV
    assert dsa.LIB.dsa_workspace_size(99, ctypes.byref(ind.struct), None, 0, 0, 2048,
                                      ctypes.byref(out)) == INV
    for k in (0, 2049):
        assert dsa.LIB.dsa_workspace_size(dsa.DSA_OP_SELECT, ctypes.byref(ind.struct), None, 0,
                                          0, k, ctypes.byref(out)) == INV
    assert dsa.LIB.dsa_workspace_size(dsa.DSA_OP_SELECT, None, None, 0, 0, 2048,
                                      ctypes.byref(out)) == INV
    # the paged score block is bounded like the contiguous one: 1000 sequences
    # of up to 128K keys keep 148-row blocks of at most 80 MiB, not n_q rows
    pind = dsa._Keep(_indexer(dsa, _paged(dsa), 1000, 0), [])
    sel = dsa.dsa_workspace_size(dsa.DSA_OP_SELECT, pind, None, 0, 0, 2048)
    assert sel <= (80 << 20) and (sel // (2048 * 64 * 4)) % 148 == 0


def test_noalloc_checks(dsa):
    ind = _indexer(dsa)
    INV = dsa.DSA_ERR_INVALID_ARG
    call = dsa.LIB.dsa_select_noalloc
    _expect(dsa, INV, lambda: call(None, 2048, _p(FAKE), 2048, None))
    _expect(dsa, INV, lambda: call(ctypes.byref(ind), 2048, None, 2048, None))
    _expect(dsa, INV, lambda: call(ctypes.byref(ind), 0, _p(FAKE), 2048, None))
    _expect(dsa, INV, lambda: call(ctypes.byref(ind), 2048, _p(FAKE), 2000, None))
    big = _mut(ind, n_keys=(16 << 20) // 4 + 1)
    _expect(dsa, dsa.DSA_ERR_WORKSPACE_TOO_SMALL,
            lambda: call(ctypes.byref(big), 2048, _p(FAKE), 2048, None))


def test_kl_and_select_scored_checks(dsa):
    ind, att = _indexer(dsa), _attn(dsa)
    INV, UNS, WS = dsa.DSA_ERR_INVALID_ARG, dsa.DSA_ERR_UNSUPPORTED, \
        dsa.DSA_ERR_WORKSPACE_TOO_SMALL
    P = FAKE + 0x200000

    def kl(attn=att, idx=P, ld_idx=2048, k=2048, lse=P, sel=P, ld_sel=2048, loss=P, grad=P,
           ld_grad=2048):
        return dsa.LIB.dsa_indexer_kl(ctypes.byref(attn), _p(idx), ld_idx, k, _p(lse), _p(sel),
                                      ld_sel, _p(loss), _p(grad), ld_grad, None)
    _expect(dsa, dsa.DSA_ERR_CUDA, lambda: kl())
    for kw in (dict(idx=None), dict(lse=None), dict(sel=None), dict(loss=None), dict(grad=None),
               dict(k=0), dict(k=2049), dict(ld_idx=100), dict(ld_sel=100), dict(ld_grad=100)):
        _expect(dsa, INV, lambda: kl(**kw))
    f32 = _mut(att, dtype=dsa.DSA_F32, heads=8, d_qk=64, d_v=64, ld_q=512, ld_kv=64)
    _expect(dsa, UNS, lambda: kl(attn=f32))

    def ss(k=2048, idx=P, ld_idx=2048, sel=P, ld_sel=2048, ws=FAKE + 0x100000, ws_bytes=1 << 34):
        return dsa.LIB.dsa_select_scored(ctypes.byref(ind), k, _p(idx), ld_idx, _p(sel), ld_sel,
                                         _p(ws), ws_bytes, None)
    _expect(dsa, dsa.DSA_ERR_CUDA, lambda: ss())
    for kw in (dict(idx=None), dict(sel=None), dict(k=0), dict(ld_idx=1), dict(ld_sel=1)):
        _expect(dsa, INV, lambda: ss(**kw))
    _expect(dsa, WS, lambda: ss(ws_bytes=1024))
    _expect(dsa, WS, lambda: ss(ws=None))

    def dense(attn=att, out=FAKE + 0x2000):
        return dsa.LIB.dsa_dense_mqa_fwd(ctypes.byref(attn), _p(out), None, None)
    _expect(dsa, dsa.DSA_ERR_CUDA, lambda: dense())
    _expect(dsa, INV, lambda: dense(out=None))
    _expect(dsa, INV, lambda: dense(out=FAKE + 0x2004))
    _expect(dsa, UNS, lambda: dense(attn=_mut(f32, n_keys=5000, n_q=100)))   # fp32 dense > 4096 keys


def test_backward_checks(dsa):
    att = _attn(dsa)
    INV, UNS = dsa.DSA_ERR_INVALID_ARG, dsa.DSA_ERR_UNSUPPORTED
    P = FAKE + 0x200000

    def bwd(attn=att, idx=P, ld_idx=2048, k=2048, out=P + 0x1000, lse=P, d_out=P + 0x2000,
            d_q=P + 0x3000, d_kv=P, ld_dkv=576, delta=P):
        return dsa.LIB.dsa_sparse_mqa_bwd(ctypes.byref(attn), _p(idx), ld_idx, k, _p(out),
                                          _p(lse), _p(d_out), _p(d_q), _p(d_kv), ld_dkv,
                                          _p(delta), None)
    _expect(dsa, dsa.DSA_ERR_CUDA, lambda: bwd())
    for kw in (dict(idx=None), dict(out=None), dict(lse=None), dict(d_out=None), dict(d_q=None),
               dict(d_kv=None), dict(delta=None), dict(k=0), dict(k=2049), dict(ld_idx=100),
               dict(ld_dkv=575), dict(out=P + 0x1008), dict(d_out=P + 0x2008),
               dict(d_q=P + 0x3004)):
        _expect(dsa, INV, lambda: bwd(**kw))
    f32 = _mut(att, dtype=dsa.DSA_F32, heads=8, d_qk=64, d_v=64, ld_q=512, ld_kv=64)
    _expect(dsa, UNS, lambda: bwd(attn=f32))
    _expect(dsa, UNS, lambda: bwd(attn=_attn(dsa, kv=_paged(dsa), n_q=64)))


def test_nvtx_ranges_switch_on_without_a_profiler():
    """DSA_NVTX=1 turns the per-call and per-block NVTX ranges on (read once
    per process); with no profiler attached they are no-ops and the call
    behaves as before."""
    import subprocess
    import sys
    code = (
        "import ctypes, sys; sys.path.insert(0, %r)\n"
        "from sparse_attention_long_tcgen05_b200 import dsa\n"
        "import test_abi_checks as t\n"
        "ind, att = t._indexer(dsa), t._attn(dsa)\n"
        "st = t._forward(dsa, ind, att)\n"
        "print(st)\n") % (os.path.dirname(os.path.dirname(os.path.abspath(__file__))),)
    env = dict(os.environ, DSA_NVTX="1",
               PYTHONPATH=os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip().splitlines()[-1] == str(4)   # DSA_ERR_CUDA: no device here
