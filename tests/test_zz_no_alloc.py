"""g4attn_decode_noalloc, the decode entry point for callers that cannot allocate device
memory (for example a plugin whose host framework owns every device allocation and hands it
only input and output buffers).  It keeps its split partials in a fixed scratch array inside
the library.  This file sorts last so a run that stops at the first failure has run every
other test before it; it also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

from attention_g4attn_b200 import synth, workloads
from parity import assert_parity, to_np

pytestmark = pytest.mark.gpu


def _binding():
    from attention_g4attn_b200 import binding
    return binding


@pytest.mark.parametrize("B,L,seed", [(16, 4096, 31)])
def test_noalloc_decode_matches_workspace_decode_on_two_calls(B, L, seed):
    b = _binding()
    dev = torch.device("cuda:0")
    ly = workloads.GLOBAL_8TO1
    cfg = b.LayerCfg.from_layer(ly)
    # two calls in a row on different inputs: the second must not see the first's partials
    for call, (bb, ll) in enumerate([(B, L), (B // 2, L + 777)]):
        d = synth.decode_inputs(bb, ll, ly.n_q_heads, ly.n_kv_heads, ly.head_dim, False,
                                seed=seed + call)
        q, k = d.q.to(dev), d.k.to(dev)
        ref, ref_lse = b.g4attn_decode(q, k, None, cfg, want_lse=True)
        got, got_lse = b.g4attn_decode_noalloc(q, k, None, cfg, want_lse=True)
        torch.cuda.synchronize()
        assert b.g4attn_device_status() == 0
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
