"""Host-side checks of the row-sharded plan (no GPU: these calls stop before any
device work): argument errors, the workspace it asks for, and the row split of the
binding."""
import ctypes

import pytest

import rank_orthonormalized_optimizer_b200 as dion


def _init(buckets, shards, **kw):
    descs = (dion.BucketDesc * len(buckets))()
    for i, (c, m, n, r) in enumerate(buckets):
        descs[i].count, descs[i].m, descs[i].n, descs[i].r, descs[i].scale = c, m, n, r, 0.0
    sh = (dion.ShardDesc * len(shards))()
    for i, (m_full, row0) in enumerate(shards):
        sh[i].m_full, sh[i].row0 = m_full, row0
    o = dion.default_options()
    for k, v in kw.items():
        setattr(o, k, v)
    h = ctypes.c_void_p()
    ws = ctypes.c_size_t()
    code = dion.dion_init_sharded(descs, sh, len(buckets), ctypes.byref(o), ctypes.byref(h),
                                  ctypes.byref(ws))
    if code == dion.OK:
        dion.dion_free(h)
    return code, ws.value


@pytest.mark.parametrize("bucket,shard,code", [
    ((2, 128, 128, 32), (256, 0), dion.OK),
    ((2, 128, 128, 32), (256, 128), dion.OK),
    ((2, 100, 136, 128), (200, 100), dion.OK),          # r above the local rows, below m_full
    ((2, 128, 128, 32), (256, 129), dion.ERR_INVALID_ARG),   # rows past the matrix
    ((2, 128, 128, 32), (256, -1), dion.ERR_INVALID_ARG),
    ((2, 128, 128, 32), (100, 0), dion.ERR_INVALID_ARG),     # more local rows than m_full
    ((2, 100, 136, 144), (200, 0), dion.ERR_UNSUPPORTED_SHAPE),  # r > n
    ((2, 8, 128, 32), (16, 0), dion.ERR_UNSUPPORTED_SHAPE),      # r > m_full
])
def test_sharded_init_checks(bucket, shard, code):
    assert _init([bucket], [shard])[0] == code


def test_sharded_plans_run_on_the_tensor_path_only():
    assert _init([(2, 128, 128, 32)], [(256, 0)], kernel_path=1)[0] == dion.ERR_INVALID_ARG
    assert b"tensor path" in dion.dion_last_error()


def test_sharded_workspace_holds_the_gather():
    """The sharded plan adds, per bucket, three [count, m_full, r] fp32 arrays (the
    gathered P0 and Householder QR's two work arrays) to what a plan of its local rows
    needs."""
    code, ws_sh = _init([(2, 512, 256, 64)], [(2048, 512)])
    assert code == dion.OK
    plain = dion.DionB200([(2, 512, 256, 64)])
    gather = 3 * 2 * 2048 * 64 * 4
    assert ws_sh >= plain.workspace_bytes + gather
    assert ws_sh <= plain.workspace_bytes + gather + 8 * 1024    # alignment only


def test_continue_without_a_step_is_refused():
    h = dion.DionB200RowSharded([(2, 256, 128, 32)], 0, 2)
    x = dion.Exchange()
    assert dion.dion_step_sharded_continue(h._h, ctypes.byref(x)) == dion.ERR_INVALID_ARG
    assert x.count == 0
    assert dion.dion_step_sharded_continue(None, ctypes.byref(x)) == dion.ERR_NOT_INITIALIZED


@pytest.mark.parametrize("m,world", [(256, 2), (11008, 3), (37, 4), (4096, 8)])
def test_binding_row_split_covers_every_row_once(m, world):
    rows = [dion.row_range(m, world, k) for k in range(world)]
    assert rows[0][0] == 0 and sum(k for _, k in rows) == m
    for (a0, ak), (b0, _) in zip(rows, rows[1:]):
        assert a0 + ak == b0
    hs = [dion.DionB200RowSharded([(1, m, 64, 16)], k, world) for k in range(world)]
    assert [h.shapes[0].m for h in hs] == [k for _, k in rows]
