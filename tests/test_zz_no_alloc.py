"""zha_attend_noalloc, the attention entry point that allocates nothing.

Callers that cannot let a library allocate device memory once they run (a server
that gives all GPU memory to its own pool at start-up, a latency-critical loop that
cannot take the synchronisation cudaMalloc / cudaFree may cause) call
zha_attend_noalloc instead of zha_attend: same arguments, same kernels, with the
scratch taken from a 32 MiB static device array of the library. These tests call
it through the C ABI and check, on calls in a row with different walk counts,
selections and output types, that it gives what zha_attend gives, that the calls
after the first change the device's free memory by nothing, and that a call
needing more than the array holds is refused before anything is launched. The
third call has more than 2,048 walks, which takes the attention's separate plan
kernel, right after smaller calls have left their plans in the array.

The file is named to be collected last, so that a run stopping at the first
failure has run every other test before it.
"""
import pytest
import torch

import synthetic as S
from helpers import attn_tol

pytestmark = pytest.mark.gpu

W_SMALL = S.scaled(S.WORKLOADS["kv256k"], name="kv256k_noalloc", batch=4, n_keys=32768 + 5 * 8 + 3, depth=5,
                   appends=0)


def zha():
    import tree_indexed_sparse_append_b200 as Z

    return Z


def queries(w, inp, n_q: int) -> torch.Tensor:
    """n_q queries per query head, drawn with the workload's recipe."""
    wq = S.scaled(w, queries_per_head=n_q)
    group = w.n_q_heads // w.n_kv_heads
    Q = torch.empty(w.batch, w.n_q_heads, n_q, w.d, dtype=inp.Q.dtype, device="cuda")
    for b in range(w.batch):
        for hq in range(w.n_q_heads):
            q, _ = S.draw_queries(wq, inp.centres[b, hq // group], b, hq, device="cuda")
            Q[b, hq] = q
    return Q


def noalloc(Z, tree, Q, sel, cnt, out, lse) -> int:
    B, Hq, nq, d = Q.shape
    code = {torch.float32: Z.F32, torch.bfloat16: Z.BF16}
    return Z.lib().zha_attend_noalloc(tree._h, Q.data_ptr(), code[Q.dtype], Hq, nq, sel.data_ptr(), cnt.data_ptr(),
                                      sel.shape[1], out.data_ptr(), code[out.dtype], lse.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)


def assert_same(out, lse, ref_out, ref_lse, atol, what):
    g, r = out.double().cpu(), ref_out.double().cpu()
    bad = (g - r).abs() > atol * r.abs().clamp(min=1.0)
    assert not bad.any(), f"{what}: {int(bad.sum())} output elements differ, max {float((g - r).abs().max())}"
    gl, rl = lse.double().cpu(), ref_lse.double().cpu()
    finite = torch.isfinite(rl)
    assert torch.equal(torch.isfinite(gl), finite), what
    assert ((gl - rl)[finite].abs() <= atol * rl[finite].abs().clamp(min=1.0)).all(), f"{what}: lse differs"


def test_noalloc_matches_attend_on_two_calls():
    Z = zha()
    w = W_SMALL
    inp = S.draw(w, device="cuda")
    tree = Z.Tree(inp.K, inp.V, inp.refs, w.n_keys, w.chunk, w.depth, w.beta, w.top_width)
    atol = attn_tol(w)
    calls = [  # (queries per head, mode, p, k, output dtype): consecutive calls differ in every one
        (1, Z.TOP_P, 0.9, 0, torch.float32),
        (3, Z.TOP_K, 0.0, 8, torch.bfloat16),
        (48, Z.TOP_P, 0.9, 0, torch.float32),  # 3,072 walks: the plan-kernel path
    ]
    for i, (n_q, mode, p, k, out_dtype) in enumerate(calls):
        Q = queries(w, inp, n_q)
        sel, cnt, _ = tree.search(Q, mode, p, k)
        ref_out, ref_lse = tree.attend(Q, sel, cnt, out_dtype=out_dtype)
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        rc = noalloc(Z, tree, Q, sel, cnt, out, lse)
        assert rc == Z.OK, Z.lib().zha_last_error()
        torch.cuda.synchronize()
        free_after = torch.cuda.mem_get_info()[0]
        tree.sync_status()
        if i > 0:  # the first call on a device may load the library's module; later ones allocate nothing
            assert free_after == free_before, (free_before, free_after)
        assert_same(out, lse, ref_out, ref_lse, atol, f"call {i + 1}")
    tree.close()


def test_noalloc_refuses_more_than_its_scratch():
    Z = zha()
    w = W_SMALL
    inp = S.draw(w, device="cuda")
    tree = Z.Tree(inp.K, inp.V, inp.refs, w.n_keys, w.chunk, w.depth, w.beta, w.top_width)
    # 32,768 walks (512 queries per head) need 43.5 MB of scratch at d = 128
    n_q = 512
    Q = queries(w, inp, n_q)
    walks = w.batch * w.n_q_heads * n_q
    sel = torch.zeros(walks, 1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(walks, dtype=torch.int32, device="cuda")
    out = torch.zeros(w.batch, w.n_q_heads, n_q, w.d, dtype=torch.float32, device="cuda")
    lse = torch.zeros(walks, dtype=torch.float32, device="cuda")
    launches = Z.kernel_launches()
    rc = noalloc(Z, tree, Q, sel, cnt, out, lse)
    assert rc == Z.ERR_CAPACITY
    assert b"scratch" in Z.lib().zha_last_error()
    assert Z.kernel_launches() == launches
    # half the walks fit
    rc = noalloc(Z, tree, Q[:, :, : n_q // 2].contiguous(), sel[: walks // 2], cnt[: walks // 2],
                 out[:, :, : n_q // 2].contiguous(), lse[: walks // 2])
    assert rc == Z.OK, Z.lib().zha_last_error()
    torch.cuda.synchronize()
    tree.close()
