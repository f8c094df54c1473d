"""Column-parallel sharding run through the product on one GPU: a layer is
split with shard_rows, each shard's rows of W, bitmap and pattern ids are
packed with patch_pack and multiplied with patch_gemm, and the shards' outputs
concatenated along N must match the oracle on the whole layer (the layer's
tolerance) -- the chain shard_rows -> shard_of -> patch_pack -> patch_gemm
that each GPU of a sharded job runs on its own rows."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
import tile_sparse_gemm_b200 as tsg
from _util import bits_of, check_gemm, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n_shards", [2, 3])
@pytest.mark.parametrize("tiles", ["clustered", "exact"])
def test_shards_through_pack_and_gemm_concatenate_to_the_layer(n_shards, tiles):
    N, K = 128 * 11, 128 * 6
    w = si.gen_w(N, K, 16, n_shards)
    bm = {"clustered": si.tiles_clustered, "exact": si.tiles_exact}[tiles](N, K, 0.5, 16, n_shards)
    ids = si.patterns_top2(w)
    wd, bmd, idd = to_dev_bf16(w), to_dev(bm), to_dev(ids)
    rows = tsg.shard_rows(bm, n_shards)
    status = tsg.new_status()
    packs = []
    for r in rows:
        ws, bs, is_ = tsg.shard_of(wd, bmd, idd, r)
        packs.append(tsg.patch_pack(ws.contiguous(), bs.contiguous(), is_.contiguous(), status=status))
    assert sum(p.N for p in packs) == N
    for M in (1, 5, 16, 300):  # both decode paths' token range and the prefill path
        x = si.gen_x(M, K, 16, M)
        xd = to_dev_bf16(x)
        y = torch.cat([tsg.patch_gemm(xd, p, status=status) for p in packs], dim=1)
        code, bits = tsg.patch_read_status(status)
        assert code == 0, (code, bits)
        check_gemm(bits_of(y), oracle.hybrid_gemm(x, w, bm, ids), f"{n_shards} shards, {tiles}, M={M}")
