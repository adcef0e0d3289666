"""The 40-layer decode schedule: its structure and per-token byte count on the
host, and one whole-model step against the oracle on the GPU.

Every layer of every cache is checked like a single-cache step: packed bytes
are exact, the index stages match the oracle up to allowed boundary swaps
(conditionally on the GPU's block set), and each layer's attention output is
within the attention tolerance.  SWA-only layers attend to their window
alone."""
import pytest
import torch

import synth
from parity_util import OracleRequest, check_step


def test_schedule40_layout_and_bytes():
    s = synth.schedule40(small=True)
    assert s.n_layers == 40
    modes = [m for c in s.caches for m in c.layers]
    assert modes[:2] == ["swa", "swa"]
    assert modes[2:20] == (["full"] + ["reuse"] * 5) * 3
    assert modes[20:24] == ["full", "reuse", "reuse", "reuse"]
    assert modes[24:] == ["reindex", "reuse", "reuse", "reuse"] * 4
    # four KV-producing layers: three m=2 encoder caches and one m=1 decoder cache
    producing = [c for c in s.caches if c.index != "none"]
    assert [c.m[0] for c in producing] == [2, 2, 2, 1]
    # 416 B per entry (288 B FP4 row + 128 B FP8 key): 3 x 416/2 + 416 per context token
    assert s.kv_bytes_per_token() == 1040.0
    # every cache appends one token per step
    assert all(c.n_new == [1] * c.batch for c in s.caches)


@pytest.mark.gpu
def test_schedule40_step_matches_oracle():
    from csa2_sparse_attention_decode_b200.harness import ScheduleWorkload

    s = synth.schedule40(small=True)
    sw = ScheduleWorkload(s, out_fp32=True)
    for w, dw in zip(s.caches, sw.parts):
        refs = [OracleRequest(w, b, w.n_tok[b] + w.n_new[b]) for b in range(w.batch)]
        check_step(w, dw, refs)
    torch.cuda.synchronize()
