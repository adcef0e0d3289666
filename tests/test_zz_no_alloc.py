"""csa2_attend_noalloc -- attention for callers that cannot allocate device
memory: code inside a host framework that owns all device memory and gives
plugins no allocator, or a serving loop that must not allocate once it runs
(an allocation can synchronise the device).  It keeps its split partials in
a fixed array inside the library instead of a caller workspace.

Each call is checked element by element against the oracle's attention over
the same top-k and window (the parity tolerance) and against csa2_attend's
output (the same tolerance), on two calls in a row: the shared array keeps the
previous call's contents, which must not leak into the next.  Cases cover a
partial head group (40 heads), the most heads (128), both output types and a
batch that fills every row of the array.  This file is collected last on
purpose."""
import pytest
import torch

import synth
from parity_util import ATOL, RTOL, OracleRequest, bits, check_attention

pytestmark = pytest.mark.gpu

CASES = [
    # name, heads, batch, out_fp32, layers
    ("H64-B2-fp32", 64, 2, True, ["full", "reuse", "reuse", "reindex", "reuse"]),
    ("H40-B3-bf16", 40, 3, False, ["full", "reuse"]),
    ("H128-B2-fp32", 128, 2, True, ["full", "reuse"]),
    ("H128-B4-bf16-full-array", 128, 4, False, ["full", "reuse"]),   # batch * heads == the limit
]


def _bf16_tol(ref):
    half_ulp = torch.from_numpy(ref).float().to(torch.bfloat16).float().abs()
    return torch.ldexp(torch.ones_like(half_ulp), torch.frexp(half_ulp.clamp_min(1e-30))[1] - 9)


@pytest.mark.parametrize("name,heads,batch,out_fp32,layers", CASES, ids=[c[0] for c in CASES])
def test_noalloc_attend_matches_oracle_and_workspace_attend(name, heads, batch, out_fp32, layers):
    import csa2_sparse_attention_decode_b200 as csa2
    from csa2_sparse_attention_decode_b200.harness import SOFTMAX_SCALE, DeviceWorkload

    assert batch * heads <= csa2.ATTEND_NOALLOC_MAX_ROWS
    n_tok = [5000 + 1700 * b for b in range(batch)]
    w = synth.Workload(f"noalloc-{name}", 21 + heads, batch, heads, n_tok, [1 + (b % 2) for b in range(batch)],
                       "hier", layers, False)
    dw = DeviceWorkload(w, out_fp32=out_fp32)
    dw.step()                                    # top-k and reference outputs through csa2_attend
    torch.cuda.synchronize()
    assert csa2.csa2_get_device_error(dw.cache) == 0
    refs = [OracleRequest(w, b, w.n_tok[b]) for b in range(batch)]
    for li in (len(layers) - 1, 1):              # two calls in a row, different queries (and groups)
        q = dw.layers[li][0]
        topk = dw.topk[dw.layer_topk[li]]
        out = torch.full_like(dw.outs[li], float("nan"))
        assert csa2.csa2_attend_noalloc(dw.cache, q, topk, SOFTMAX_SCALE, out) == 0
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        for b in range(batch):
            r = refs[b].attend(bits(q[b]), topk[b].cpu().numpy(), SOFTMAX_SCALE)
            check_attention(out[b], r, f"{name} layer {li} request {b}: noalloc vs oracle")
        ref = dw.outs[li].float()
        tol = ATOL + RTOL * ref.abs()
        if not out_fp32:
            tol = tol + 2 * _bf16_tol(ref.cpu().numpy()).to(ref.device)   # each side rounds once to bf16
        assert ((out.float() - ref).abs() <= tol).all(), f"{name} layer {li}: noalloc vs csa2_attend"
    assert csa2.csa2_get_device_error(dw.cache) == 0


def test_noalloc_attend_rejects_sizes_over_its_limit():
    import csa2_sparse_attention_decode_b200 as csa2
    from csa2_sparse_attention_decode_b200.harness import SOFTMAX_SCALE, DeviceWorkload

    w = synth.workload(4, small=True)            # 8 requests
    dw = DeviceWorkload(w, build=False)
    heads = csa2.ATTEND_NOALLOC_MAX_ROWS // w.batch + 1
    q = torch.zeros(w.batch, heads, 512, dtype=torch.bfloat16, device="cuda")
    topk = torch.full((w.batch, 512), -1, dtype=torch.int32, device="cuda")
    out = torch.zeros(w.batch, heads, 512, dtype=torch.float32, device="cuda")
    assert csa2.csa2_attend_noalloc(dw.cache, q, topk, SOFTMAX_SCALE, out) == 2
