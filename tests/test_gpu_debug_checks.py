"""Debug aids on the GPU.

  * kv8_check_indices counts out-of-range context lengths, block-table
    entries a decode would read, and slots, exactly; the errors are planted
    on the host into copies of a workload's indices, and only the check
    kernels (which read nothing but those arrays) ever see them;
  * guard bytes: the decode calls (INT8 split and unsplit, fused append,
    KIVI) write nothing before or after `out` and the workspace, and the
    appends write no page record or tail row they do not own.
"""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU machine
    pytest.skip("needs a GPU", allow_module_level=True)

from tests import gpu_util as U  # noqa: E402

GUARD = 4096  # bytes on each side


@pytest.fixture(scope="module")
def pk():
    from paged_int8_kv_b200 import build
    build.build()
    import paged_int8_kv_b200 as m
    yield m
    assert m.kv8_read_device_status(clear=True) == 0


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def test_check_indices_counts_planted_errors(pk):
    w = W.tiny()  # rows of 16 entries; sequence 1 (200 tokens) reads 13
    bt, cl, nb, mcl = w.block_tables, w.context_lens, w.num_blocks, w.max_context_len

    def check(bt_, cl_):
        return pk.kv8_check_indices(_dev(bt_), _dev(cl_), mcl, nb)
    assert check(bt, cl) == (0, 0, 0)
    bt2 = bt.copy()
    bt2[0, 3] = nb        # read, past the last block
    bt2[1, 0] = -5        # read, negative
    bt2[1, 15] = -1       # past sequence 1's 13 pages: never read
    assert check(bt2, cl) == (0, 2, 0)
    cl2 = cl.copy()
    cl2[1] = -3           # a bad length; its row is then not scanned
    assert check(bt2, cl2) == (1, 1, 0)
    cl3 = cl.copy()
    cl3[0] = mcl + 16     # longer than the bound; the scan stops at the bound
    assert check(bt, cl3) == (1, 0, 0)
    sm = np.array([0, 5, -1, nb * 16 - 1, nb * 16, nb * 16 + 7, -9], np.int64)
    assert pk.kv8_check_indices(None, None, 0, nb, slot_mapping=_dev(sm)) == (0, 0, 2)
    assert pk.kv8_check_indices(_dev(bt2), _dev(cl2), mcl, nb,
                                slot_mapping=_dev(sm)) == (1, 1, 2)


def _guarded(nbytes, fill):
    raw = torch.full((GUARD + nbytes + GUARD,), fill, dtype=torch.uint8, device="cuda")
    return raw, raw[GUARD:GUARD + nbytes]


def _guards_intact(raw, fill):
    g = raw.cpu().numpy()
    return bool(np.all(g[:GUARD] == fill) and np.all(g[-GUARD:] == fill))


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("chunk", [0, 64])
def test_decode_writes_stay_in_out_and_workspace(pk, out_dtype, chunk):
    w = W.tiny()
    cache, q, bt, cl = U.device_inputs(w)
    esize = 4 if out_dtype == torch.float32 else 2
    raw_o, out_b = _guarded(q.numel() * esize, 0xA5)
    out = out_b.view(out_dtype).view(q.shape)
    nws = pk.kv8_decode_workspace_bytes(w.batch, w.num_q_heads, 128, w.max_context_len, chunk)
    raw_w, ws = _guarded(max(nws, 16), 0x5A)
    pk.kv8_paged_decode_attention(q, cache.k_cache, cache.v_cache, cache.k_scales,
                                  cache.v_scales, bt, cl, out, w.max_context_len,
                                  chunk_tokens=chunk, workspace=ws)
    ref = torch.empty(q.shape, dtype=out_dtype, device="cuda")
    ws2 = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
    pk.kv8_paged_decode_attention(q, cache.k_cache, cache.v_cache, cache.k_scales,
                                  cache.v_scales, bt, cl, ref, w.max_context_len,
                                  chunk_tokens=chunk, workspace=ws2)
    torch.cuda.synchronize()
    assert _guards_intact(raw_o, 0xA5) and _guards_intact(raw_w, 0x5A)
    assert torch.equal(out.view(torch.int16 if esize == 2 else torch.int32),
                       ref.view(torch.int16 if esize == 2 else torch.int32))


def test_fused_append_writes_only_the_new_slots(pk):
    from paged_int8_kv_b200 import PagedKV8Cache
    from paged_int8_kv_b200.runtime import fill_from_host
    w = W.tiny()
    c = PagedKV8Cache(w.num_blocks, w.num_kv_heads, device="cuda")
    fill_from_host(c, w.fill_segments())
    before = [t.clone() for t in (c.k_cache, c.v_cache, c.k_scales, c.v_scales)]
    kn, vn, sl = w.step_tokens()
    q = _dev(w.q()).view(torch.bfloat16)
    raw_o, out_b = _guarded(q.numel() * 4, 0xC3)
    out = out_b.view(torch.float32).view(q.shape)
    nws = pk.kv8_decode_workspace_bytes(w.batch, w.num_q_heads, 128, w.max_context_len, 64)
    raw_w, ws = _guarded(max(nws, 16), 0x3C)
    pk.kv8_paged_decode_attention_append(q, _dev(kn).view(torch.bfloat16),
                                         _dev(vn).view(torch.bfloat16), c.k_cache,
                                         c.v_cache, c.k_scales, c.v_scales,
                                         _dev(w.block_tables), _dev(w.context_lens),
                                         out, w.max_context_len, chunk_tokens=64,
                                         workspace=ws)
    torch.cuda.synchronize()
    assert _guards_intact(raw_o, 0xC3) and _guards_intact(raw_w, 0x3C)
    # only the step's slots changed (the rows and scales of those tokens)
    slots = sl[sl >= 0]
    mask = np.zeros(w.num_blocks * 16, bool)
    mask[slots] = True
    mask = mask.reshape(w.num_blocks, 16)
    for old, new in zip(before, (c.k_cache, c.v_cache, c.k_scales, c.v_scales)):
        o, n = old.cpu().numpy(), new.cpu().numpy()
        keep = ~mask[:, None, :]  # [NB, 1, 16] over heads
        if o.ndim == 4:
            keep = keep[..., None]
        same = (o.view(np.uint8) == n.view(np.uint8)) if o.dtype == np.int8 else (
            o.view(np.uint32) == n.view(np.uint32))
        assert np.all(same | ~np.broadcast_to(keep, same.shape))


def test_kivi_writes_stay_in_owned_records(pk):
    w = W.make_workload("kivi_guard", 2401, [15, 16, 33, 0, 47], 8, 2, extra_blocks=6)
    REC = pk.KV8_KIVI_PAGE_BYTES
    raw_c, cache_b = _guarded(w.num_blocks * w.num_kv_heads * REC, 0x77)
    cache = cache_b.view(w.num_blocks, w.num_kv_heads, REC)
    tail_bytes = w.batch * w.num_kv_heads * 2 * 16 * 128 * 2
    raw_t, tail_b = _guarded(tail_bytes, 0x66)
    tail = tail_b.view(torch.bfloat16).view(w.batch, w.num_kv_heads, 2, 16, 128)
    bt = _dev(w.block_tables)
    for k, v, cu, cl in list(w.kivi_fill_calls()) + [w.kivi_step_call()]:
        pk.kv8_kivi_append(_dev(k).view(torch.bfloat16), _dev(v).view(torch.bfloat16),
                           _dev(cu), _dev(cl), bt, cache, tail,
                           max(int(np.diff(cu).max(initial=0)), 1))
    torch.cuda.synchronize()
    assert _guards_intact(raw_c, 0x77) and _guards_intact(raw_t, 0x66)
    # records of blocks that hold no full page are untouched
    full = set()
    for b, t in enumerate(w.context_lens):
        full.update(int(x) for x in w.block_tables[b, :int(t) // 16])
    c = cache.cpu().numpy()
    for blk in range(w.num_blocks):
        if blk not in full:
            assert np.all(c[blk] == 0x77), blk
    # tail rows no call's partial page held are untouched: the fill call
    # leaves rows 0 .. (T-2) % 16 when T - 1 is not a multiple of 16, and the
    # step's last token goes to row (T-1) % 16 unless it completes its page
    tv = tail_b.cpu().numpy().reshape(w.batch, w.num_kv_heads, 2, 16, 256)
    for b, t in enumerate(int(x) for x in w.context_lens):
        hi = -1 if t == 0 else ((t - 1) % 16 if t % 16 else 14)
        assert np.all(tv[b, :, :, hi + 1:] == 0x66), b
    # the decode writes only `out`
    q = _dev(w.q()).view(torch.bfloat16)
    raw_o, out_b = _guarded(q.numel() * 4, 0x11)
    out = out_b.view(torch.float32).view(q.shape)
    nws = pk.kv8_decode_workspace_bytes(w.batch, w.num_q_heads, 128, w.max_context_len, 16)
    raw_w, ws = _guarded(max(nws, 16), 0x22)
    pk.kv8_kivi_paged_decode_attention(q, cache, tail, bt, _dev(w.context_lens), out,
                                       w.max_context_len, chunk_tokens=16, workspace=ws)
    torch.cuda.synchronize()
    assert _guards_intact(raw_o, 0x11) and _guards_intact(raw_w, 0x22)
