"""The vocab-sharded head on CPU: two gloo ranks (world size 2, 127.0.0.1) each take their
stripe of a small FP8 head, compute its logits with the oracle, all-gather the stripes and
assemble them; the result must equal the unsharded oracle bit for bit (a row's logits are
independent of the others).  A head whose row count does not divide by the world size checks
the zero-padded last stripe.  Also the host rules of the split itself."""

import json
import os
import sys

import pytest

from decode_lm_head_b200 import shard
from test_bench_ranks import _launch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, os, sys
sys.path.insert(0, os.environ["DLMH_ROOT"])
sys.path.insert(0, os.path.join(os.environ["DLMH_ROOT"], "tests"))
import numpy as np, torch
import bench
from decode_lm_head_b200 import shard, synth
from oracle import gemv as og
world, rank, _ = bench.dist_setup(None, backend="gloo")
res = {}
for n in (1000, 1001):
    k, m = 256, 5
    w = synth.to_numpy_bits(synth.fp8_weight(n, k, 9))
    s = synth.to_numpy_bits(synth.row_scales(n, 9))
    x = synth.to_numpy_bits(synth.bf16_rows(m, k, 9))
    a, b = shard.stripe(n, world, rank)
    local = torch.zeros(m, shard.stripe_width(n, world), dtype=torch.int32)  # gloo has no 16-bit gather
    local[:, :b - a] = torch.from_numpy(og.w8a16_gemv(w[a:b], s[a:b], x).astype(np.int32))
    out = shard.gather_buffer(m, n, world, "cpu", dtype=torch.int32)
    shard.all_gather_stripes(local, out)
    full = shard.assemble(out, n).numpy().astype(np.uint16)
    res[str(n)] = bool(np.array_equal(full, og.w8a16_gemv(w, s, x)))
print(json.dumps({"rank": rank, "world": world, "equal": res}), flush=True)
import torch.distributed as dist
dist.destroy_process_group()
"""


def test_stripes_cover_the_head_in_order():
    for n in (1, 7, 1000, 1001, 248320):
        for world in (1, 2, 3, 4, 8):
            parts = [shard.stripe(n, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            assert all(parts[i][1] == parts[i + 1][0] for i in range(world - 1))
            assert all(0 <= b - a <= shard.stripe_width(n, world) for a, b in parts)
    assert shard.stripe(248320, 8, 3) == (93120, 124160)
    with pytest.raises(ValueError):
        shard.stripe(10, 2, 2)


def test_two_gloo_ranks_gather_the_unsharded_oracle_logits():
    outs = _launch(CHILD)
    lines = [json.loads(o.strip().splitlines()[-1]) for o in outs]
    assert sorted(d["rank"] for d in lines) == [0, 1]
    for d in lines:
        assert d["world"] == 2
        assert d["equal"] == {"1000": True, "1001": True}
