"""g4attn_decode_noalloc, the decode entry point for callers that cannot allocate device
memory (for example a plugin whose host framework owns every device allocation and hands it
only input and output buffers).  It keeps its split partials in a fixed scratch array inside
the library.  This file sorts last so a run that stops at the first failure has run every
other test before it; it also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

import oracle
from attention_g4attn_b200 import synth, workloads
from gpu_common import ocfg
from parity import assert_parity, to_np

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 8 << 20


def _binding():
    from attention_g4attn_b200 import binding
    return binding


def test_noalloc_decode_matches_oracle_and_workspace_decode_on_two_calls():
    """Two calls in a row on different inputs, the second larger than the first (it covers
    more of the scratch, so it cannot pass on partials the first call left).  The second
    problem (32 sequences, 32 query heads: 128 kv sequences at L=2000) needs more than the
    8 MiB scratch at the full split (two segments per sequence), so the call lowers the number
    of CTA pairs until the partials fit (64 pairs: one segment per sequence)."""
    b = _binding()
    dev = torch.device("cuda:0")
    ly = workloads.GLOBAL_8TO1
    cfg = b.LayerCfg.from_layer(ly)
    calls = [(8, 3001, 41), (32, 2000, 42)]
    assert b.g4attn_decode_workspace_size(32, 2000, cfg) > SCRATCH_BYTES   # lowering is needed
    assert b.g4attn_decode_workspace_size(8, 3001, cfg) <= SCRATCH_BYTES
    for call, (B, L, seed) in enumerate(calls):
        d = synth.decode_inputs(B, L, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False, seed=seed)
        q, k = d.q.to(dev), d.k.to(dev)
        got, got_lse = b.g4attn_decode_noalloc(q, k, None, cfg, want_lse=True)
        ref, ref_lse = b.g4attn_decode(q, k, None, cfg, want_lse=True)
        torch.cuda.synchronize()
        assert b.g4attn_device_status() == 0
        # against the fp64 oracle on sampled (batch, kv head) items
        items = np.array(sorted({0, B * ly.n_kv_heads - 1, 5, 17 % (B * ly.n_kv_heads)}),
                         np.int32)
        oo, ol = oracle.decode(d.q[:, 0], d.k, None, ocfg(ly), items=items)
        go, gl = to_np(got)[:, 0], to_np(got_lse)
        for it in items:
            bb, g = divmod(int(it), ly.n_kv_heads)
            hs = slice(g * 8, g * 8 + 8)
            assert_parity(go[bb, hs], oo[bb, hs], "noalloc vs oracle, call %d item %d" % (call, it))
            assert_parity(gl[bb, hs], ol[bb, hs], "noalloc lse vs oracle, call %d item %d" % (call, it))
        # and against the workspace decode over every sequence
        assert_parity(to_np(got), to_np(ref), "noalloc vs workspace decode, call %d" % call)
        assert_parity(to_np(got_lse), to_np(ref_lse), "noalloc lse, call %d" % call)


def test_noalloc_decode_refuses_problems_beyond_its_scratch():
    b = _binding()
    dev = torch.device("cuda:0")
    cfg = b.LayerCfg.from_layer(workloads.GLOBAL_8TO1)
    # 128 sequences x 32 heads x (512 + 2) fp32 partials need more than 8 MiB
    q = torch.zeros(128, 1, 32, 512, dtype=torch.bfloat16, device=dev)
    k = torch.zeros(128, 4, 4, 512, dtype=torch.bfloat16, device=dev)
    with pytest.raises(b.G4AttnError) as e:
        b.g4attn_decode_noalloc(q, k, None, cfg)
    assert e.value.code == b.G4ATTN_ERR_TOO_LARGE
