"""Host-side helpers of the benchmark, on the CPU."""
import hashlib

import numpy as np
import torch

import bench


def test_tensor_sha256_hashes_the_raw_bytes_of_any_dtype():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(3, 40, generator=g)
    for t in (x, x.to(torch.bfloat16), x.to(torch.float16), (x * 100).to(torch.int32)):
        raw = t.contiguous().numpy().tobytes() if t.dtype != torch.bfloat16 \
            else t.view(torch.int16).numpy().tobytes()
        assert bench.tensor_sha256(t) == hashlib.sha256(raw).hexdigest()
    a = np.arange(10, dtype=np.uint32)
    assert bench.tensor_sha256(a) == hashlib.sha256(a.tobytes()).hexdigest()
    assert bench.tensor_sha256(x.t()) == hashlib.sha256(x.t().contiguous().numpy().tobytes()).hexdigest()


def test_rank_seeds_differ_and_start_at_the_workload_seed():
    assert bench.rank_seed(0) == 5
    assert len({bench.rank_seed(r) for r in range(8)}) == 8


def test_profile_commands_use_existing_benchmark_options():
    """Every `python bench.py ...` command quoted in profiles/ parses with the
    benchmark's own options (the summaries must name commands that run)."""
    import glob
    import os
    import re
    import shlex
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmds = []
    for path in glob.glob(os.path.join(root, "profiles", "*.md")):
        text = open(path).read().replace("\\\n", " ")
        cmds += [(path, m) for m in re.findall(r"python bench\.py([^`\n]*)", text)]
    assert cmds, "no benchmark command found in profiles/"
    parser = bench.build_parser()
    for path, tail in cmds:
        args = shlex.split(tail.split(">")[0])
        parser.parse_args(args)          # SystemExit on an unknown option or kernel name


def test_group_bounds_cover_every_weight_once_in_order():
    for n, size, layers in [(224, 4, None), (224, 3, None), (224, 7, None), (10, 32, None), (224, 1, None),
                            (224, 0, [4, 1, 1, 1]), (224, 0, [3, 2, 2]), (23, 0, [3, 2, 2]), (7, 0, [7])]:
        b = bench.group_bounds(n, size, layers)
        covered = [i for lo, hi in b for i in range(lo, hi)]
        assert covered == list(range(n)), (n, size, layers)
        assert all(hi > lo for lo, hi in b)
        if layers is None:
            assert all(hi - lo <= size for lo, hi in b)
            assert len(b) == -(-n // size)
        else:
            per = sum(layers)
            # the groups repeat the layer pattern
            sizes = [hi - lo for lo, hi in b]
            assert sizes[:len(layers)] == [min(k, n) for k in layers][:len(sizes[:len(layers)])]
            assert len(b) == len(layers) * (n // per) + len([k for k in np.cumsum([0] + layers[:-1]) if k < n % per])


def test_group_bounds_reject_empty_groups():
    import pytest
    with pytest.raises(ValueError):
        bench.group_bounds(10, 0)
    with pytest.raises(ValueError):
        bench.group_bounds(10, 4, [3, 0, 4])
