"""The dense-first schedule run through the library on the GPU ("Radial
Attention", sec. 6: the first DiT blocks and the first denoising steps keep
dense attention, the rest use the radial mask).

A short schedule (3 denoising steps x 3 attention blocks, the first step and the
first block dense) runs every call through ra_attention_fwd with the mask the
policy picks, each call on its own seeded Q, K, V.  Every row of every call is
compared with the fp64 oracle under that mask, and with the oracle under the
other mask, which the output must NOT match (so the policy's choice really
reached the kernel); the dense and sparse calls are counted."""
import numpy as np
import pytest

import oracle
import synth
from tests import _gpu

pytestmark = pytest.mark.gpu

F, S, H, D = 8, 512, 1, 128       # n = 4096: the radial mask keeps 860 of 32 x 32 tiles


def test_dense_first_schedule_calls_match_the_oracle(orc):
    _gpu.need_gpu()
    ra = _gpu.ra()
    n = F * S
    sparse_mk, dense_mk = dict(family="radial"), dict(family="dense")
    sparse, dense = ra.build_mask(sparse_mk, F, S), ra.build_mask(dense_mk, F, S)
    nb = (n + 127) // 128
    assert sparse.info["nnz"] < nb * nb == dense.info["nnz"]
    specs = {id(sparse): oracle.spec_from(sparse_mk, F, S), id(dense): oracle.spec_from(dense_mk, F, S)}
    policy = ra.DenseFirstPolicy(sparse, dense, dense_steps=1, dense_blocks=1)
    steps, blocks = 3, 3
    scale = _gpu.scale_for(D)
    row_bh, row_q = _gpu.all_rows(1, H, n)
    counted = {"dense": 0, "sparse": 0}
    for t in range(steps):
        for blk in range(blocks):
            seed = 91000 + 10 * t + blk
            Qh, Kh, Vh = (synth.normal_bf16(seed, tid, (1, H, n, D)) for tid in range(3))
            m = policy.mask(t, blk)
            kind = "dense" if m is dense else "sparse"
            assert (kind == "dense") == (t < 1 or blk < 1)
            counted[kind] += 1
            q, k, v = (_gpu.to_device(x) for x in (Qh, Kh, Vh))
            o = ra.attention_fwd(q, k, v, m, scale=scale, mode="block")
            assert ra.device_status() == ra.RA_OK
            got = _gpu.gather_rows(_gpu.to_f64(o), row_bh, row_q)
            want, _, _ = orc.attention_rows(Qh, Kh, Vh, specs[id(m)], oracle.BLOCK, scale, row_bh, row_q)
            _gpu.assert_close(got, want, f"step {t} block {blk} ({kind})")
            other = dense if m is sparse else sparse
            want_other, _, _ = orc.attention_rows(Qh, Kh, Vh, specs[id(other)], oracle.BLOCK, scale, row_bh,
                                                  row_q)
            _, rel = _gpu.errors(got, want_other)
            assert rel > 20 * _gpu.REL_L2, f"step {t} block {blk}: output also matches the other mask"
    assert counted["dense"] == policy.dense_calls(steps, blocks) == 5
    assert counted["sparse"] == steps * blocks - 5
