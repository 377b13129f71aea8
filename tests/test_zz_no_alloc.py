"""The allocation-free decode indexer entry point (for callers that cannot allocate device memory,
e.g. inside an engine that owns every device allocation).  It must give the same selection as
csa_decode_index_topk with a caller workspace, on two calls in a row, and refuse requests larger
than its fixed scratch array.  Collected last on purpose."""
import numpy as np
import pytest
import torch

import synth
from tests._helpers import dev

pytestmark = pytest.mark.gpu


# the last case has rows longer than 32768 entries: the multi-block selection keeps its histograms,
# counters and candidates after the scores inside the fixed array
@pytest.mark.parametrize("Hi,P,n_cap", [(32, [4000, 4093, 2047], 1100), (8, [517, 1023, 300], 300),
                                        (32, [262000, 200003], 65536)])
def test_noalloc_matches_workspace_entry_point(Hi, P, n_cap):
    import long_context_compressed_05_b200 as h
    spec = synth.LayerSpec(kind="csa", T=0, D=256, m=4, width=8, C=256, di=64, Hi=Hi, topk=128, window=128, H=4,
                           dh=128, scale=128 ** -0.5, dtype="bf16", seed=77 + Hi)
    d = synth.DecodeSpec(layers=(spec,), B=len(P), P=max(P), seed=spec.seed)
    inp = synth.decode_inputs(d, 0, n_cap=n_cap)
    cache_t = {k: dev(inp[k]) for k in ("entries", "win_kv", "ring_g", "idx_keys", "ring_ki")}
    p = h.params_for(spec, T=0, B=len(P), n_cap=n_cap)
    cache = h.make_cache(cache_t["entries"], cache_t["win_kv"], cache_t["ring_g"], cache_t["idx_keys"],
                         cache_t["ring_ki"])
    ncols = h.hcsa_proj_cols(p, h.KIND_CSA)
    r = np.random.default_rng(5)
    y = torch.from_numpy(r.standard_normal((len(P), ncols)).astype(np.float32)).to(torch.bfloat16).cuda()
    qi = y[:, 2 * spec.C + spec.di: 2 * spec.C + spec.di + Hi * spec.di]
    w = y[:, 2 * spec.C + spec.di + Hi * spec.di: 2 * spec.C + spec.di + Hi * spec.di + Hi]
    pos = torch.tensor(P, dtype=torch.int32, device="cuda")
    ws = torch.empty(h.hcsa_workspace_bytes(p, h.OP_CSA_DECODE_INDEX_TOPK), dtype=torch.uint8, device="cuda")
    ref = torch.empty((len(P), spec.topk), dtype=torch.int32, device="cuda")
    h.csa_decode_index_topk(p, cache, pos, qi, w, ref, ws)
    for _ in range(2):
        got = torch.full_like(ref, -7)
        h.csa_decode_index_topk_noalloc(p, cache, pos, qi, w, got)
        torch.cuda.synchronize()
        assert h.hcsa_get_device_status() == 0
        assert torch.equal(got, ref)


def test_noalloc_rejects_requests_beyond_its_scratch():
    import long_context_compressed_05_b200 as h
    spec = synth.LayerSpec(kind="csa", T=0, D=256, m=4, width=8, C=256, di=64, Hi=32, topk=128, window=128, H=4,
                           dh=128, scale=0.1, dtype="bf16")
    p = h.params_for(spec, T=0, B=3, n_cap=1 << 20)       # 3 Mi scores > 2 Mi
    dummy = torch.zeros(64, dtype=torch.int32, device="cuda")
    pos = torch.zeros(3, dtype=torch.int32, device="cuda")
    qi = torch.zeros((3, spec.Hi * spec.di), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((3, spec.Hi), dtype=torch.bfloat16, device="cuda")
    sel = torch.zeros((3, spec.topk), dtype=torch.int32, device="cuda")
    # well-formed arguments: the request is refused for its size alone, before anything is launched
    cache = h.make_cache(dummy, dummy, dummy, dummy, dummy)
    with pytest.raises(h.HcsaError) as e:
        h.csa_decode_index_topk_noalloc(p, cache, pos, qi, w, sel)
    assert e.value.code == 5
    # a malformed request is refused for what is wrong with it, whatever its size
    with pytest.raises(h.HcsaError) as e:
        h.csa_decode_index_topk_noalloc(p, h.make_cache(None, None, None), pos, qi, w, sel)
    assert e.value.code == 1
    with pytest.raises(h.HcsaError) as e:
        narrow = torch.zeros((3, 64), dtype=torch.bfloat16, device="cuda")   # rows narrower than Hi * di
        h.csa_decode_index_topk_noalloc(p, cache, pos, narrow, w, sel)
    assert e.value.code == 2
    torch.cuda.synchronize()
    assert torch.count_nonzero(dummy) == 0 and torch.count_nonzero(sel) == 0
