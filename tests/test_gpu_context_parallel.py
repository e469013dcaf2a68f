"""Context-parallel decode on one GPU (through the C ABI).

Each of R emulated ranks runs kv8_paged_decode_attention_partials on its
part of every context (the tables of its shard of the same cache, as a rank
holding only those blocks would), the R partial buffers are laid out
rank-major as an all-gather leaves them, and kv8_merge_partials merges them.
The result must match the oracle over the whole contexts and the one-GPU
decode call.  Ranks are emulated one after another on the same GPU: the
kernels never wait on each other, so no emulated rank depends on another
running at the same time.
"""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU machine
    pytest.skip("needs a GPU", allow_module_level=True)

from tests import gpu_util as U  # noqa: E402


@pytest.fixture(scope="module")
def pk():
    from paged_int8_kv_b200 import build
    build.build()
    import paged_int8_kv_b200 as m
    yield m
    assert m.kv8_read_device_status(clear=True) == 0


@pytest.mark.parametrize("ranks", [1, 2, 3, 4])
@pytest.mark.parametrize("chunk", [64, 512])
def test_context_parallel_matches_oracle(pk, oracle_mod, ranks, chunk):
    from paged_int8_kv_b200 import context_parallel as CP
    lens = [5000, 1, 0, 700, 2048, 129]
    w = W.make_workload("cp", 8000 + ranks, lens, 32, 8, extra_blocks=3,
                        outliers=(3, 10.0))
    cache, q, bt, cl = U.device_inputs(w)
    maxl = CP.max_local_len(w.context_lens, ranks, chunk)
    nbytes = pk.kv8_decode_partials_bytes(w.batch, w.num_q_heads, 128, maxl, chunk)
    stride = (nbytes + 255) // 256 * 256
    allp = torch.full((ranks * stride,), 0xFF, dtype=torch.uint8, device="cuda")
    for r in range(ranks):
        t, ll, _ = CP.local_tables(w.block_tables, w.context_lens, ranks, r, chunk)
        pk.kv8_paged_decode_attention_partials(
            q, cache.k_cache, cache.v_cache, cache.k_scales, cache.v_scales,
            torch.from_numpy(t).cuda(), torch.from_numpy(ll).cuda(),
            allp[r * stride:(r + 1) * stride], maxl, chunk)
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    pk.kv8_merge_partials(allp, stride, ranks, out, maxl, chunk)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    kc, vc, ks, vs = U.oracle_full_cache(oracle_mod, w)
    ref = oracle_mod.decode_attention(w.q(), kc, vc, ks, vs, w.block_tables,
                                      w.context_lens)
    U.assert_close(got, ref, bf16=False)
    assert np.abs(got - ref).max() < 1e-4
    assert np.all(got[2] == 0.0)  # the empty context
    one = U.gpu_decode(cache, q, bt, cl, w, chunk_tokens=chunk)
    assert np.abs(got - one).max() <= 1e-5


def test_context_parallel_single_process_helper(pk, oracle_mod):
    # the plumbing entry point with world size 1 (no process group)
    from paged_int8_kv_b200 import context_parallel as CP
    w = W.make_workload("cp1", 8100, [3000, 40], 16, 4, extra_blocks=1)
    cache, q, bt, cl = U.device_inputs(w)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    CP.context_parallel_decode(q, cache.k_cache, cache.v_cache, cache.k_scales,
                               cache.v_scales, bt, cl, out, w.max_context_len,
                               256)
    torch.cuda.synchronize()
    kc, vc, ks, vs = U.oracle_full_cache(oracle_mod, w)
    ref = oracle_mod.decode_attention(w.q(), kc, vc, ks, vs, w.block_tables,
                                      w.context_lens)
    U.assert_close(out.float().cpu().numpy(), ref, bf16=True)
