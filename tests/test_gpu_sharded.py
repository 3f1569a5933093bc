"""GPU check of the row-sharded NVFP4 path on one device: the shards of a
weight are quantized one after the other through the CUDA library with the
same exchange protocol the ranks use (the all-reduce replaced by the maximum
of the shards' local maxima, which is what MAX over the ranks returns), and
the concatenated rows must equal the single-call quantization of the whole
weight byte for byte.  The multi-process exchange itself is covered on the
CPU (tests/test_multiproc_cpu.py)."""
import pytest
import torch

import fp4_post_weight_grid_b200 as fq
import synth
from fp4_post_weight_grid_b200.sharded import row_shard_protocol, shard_rows
from test_gpu_parity import DEV, _assert_eq, _np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 3, 8])
@pytest.mark.parametrize("weighted", [False, True])
def test_row_shards_equal_the_whole_weight(world, weighted):
    rows, cols = 1000, 1024
    w = synth.q_proj(rows, cols, seed=world).to(DEV)
    imp = synth.importance_diag_xtx(cols=cols, tokens=64, seed=world).to(DEV) if weighted else None
    full = fq.nvfp4_quantize(w, importance=imp)
    shards = [w[slice(*shard_rows(rows, world, r))].contiguous() for r in range(world)]
    local = []
    for x in shards:
        a = torch.empty(1, device=DEV)
        fq.fp4q_global_absmax(x, a)
        local.append(a)
    gmax = torch.stack(local).max()

    outs = []
    for x, a in zip(shards, local):
        def sweep(amax, x=x):
            n = x.shape[0]
            codes = torch.empty((n, cols // 2), dtype=torch.uint8, device=DEV)
            scales = torch.empty((n, cols // 16), dtype=torch.uint8, device=DEV)
            S = torch.empty(1, device=DEV)
            st = torch.zeros(1, dtype=torch.int32, device=DEV)
            if imp is None:
                fq.fp4q_nvfp4_sweepmse(x, amax, codes, scales, S, None, None, st)
            else:
                fq.fp4q_nvfp4_sweepwmse(x, amax, imp, codes, scales, S, None, None, st)
            return codes, scales, S, st
        outs.append(row_shard_protocol(lambda a=a: a, lambda t: t.copy_(gmax.reshape(1)), sweep))
    torch.cuda.synchronize()
    for codes, scales, S, st in outs:
        assert int(st.item()) == 0
        _assert_eq("S", _np(S), _np(full.global_scale))
    _assert_eq("codes", _np(torch.cat([o[0] for o in outs])), _np(full.codes))
    _assert_eq("scales", _np(torch.cat([o[1] for o in outs])), _np(full.scales))
