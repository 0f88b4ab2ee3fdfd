"""The scans start their set-up before the step's prologue (the one launch that
runs every layer's append jobs) has finished, and read the index query early
only when no append job writes it.  Here an append job of the step rewrites
the index query itself: the Top-K must be the one of the NEW query (checked
against the oracle by the score-tie rule), for the plain E4M3 scan and for the
MXFP4 scan."""
import numpy as np
import pytest

from oracle import indexer as oi
from oracle import mxfp4 as omx
from oracle import quant as oq
from tests.parity import topk_diff

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import indexer_selected_sparse_csa2_b200 as m
    return m


@pytest.mark.parametrize("name", ["tiny_decode", "decode_mx"])
def test_append_rewriting_the_index_query_is_seen(csa, name):
    from csa_synth import get_config
    from csa_synth.device import DeviceCase
    cfg = get_config(name)
    dc = DeviceCase(cfg)
    arr = dc.layer_descs(append_rows=True)
    dl = dc.layers[0]
    old_q = dl.qI.cpu().numpy().copy()
    rng = np.random.default_rng(11)
    qf = rng.standard_normal((cfg.B * cfg.H_I, cfg.d_I)).astype(np.float32)
    src = torch.from_numpy(qf).cuda()
    # the last append slot (the window row's job on the E4M3 layer, free on the
    # MXFP4 one): the window is not checked here, only the index
    arr[0].append[2] = csa.quant_job(src, csa.CSA_FMT_FP8_E4M3_PLAIN, dl.qI, cfg.d_I, n_rows=cfg.B * cfg.H_I)
    csa.csa_layer_step(arr)
    torch.cuda.synchronize()
    assert csa.device_status() == 0
    new_q = oq.e4m3_cast(qf).reshape(cfg.B, cfg.H_I, cfg.d_I)
    assert np.array_equal(dl.qI.cpu().numpy().reshape(cfg.B, cfg.H_I, cfg.d_I), new_q)
    w = dl.w.cpu().numpy().reshape(cfg.B, cfg.H_I)
    idx = dl.idx.cpu().numpy()
    moved = 0
    for b in (0, cfg.B - 1):
        if cfg.key_format == "mxfp4":
            ent = np.concatenate([dc.keys[0][b].cpu().numpy(), dc.key_scales[0][b].cpu().numpy()], axis=1)
            S = omx.mx_index_scores(new_q[b], w[b], ent)
            S_old = omx.mx_index_scores(old_q[b, 0], w[b], ent)
        else:
            kc = dc.keys[0][b].cpu().numpy()
            S = oi.index_scores(new_q[b], w[b], kc)
            S_old = oi.index_scores(old_q[b, 0], w[b], kc)
        want = oi.topk(S, cfg.K)
        topk_diff(idx[b, 0], want, lambda p: S[p])
        moved += not np.array_equal(np.sort(want), np.sort(oi.topk(S_old, cfg.K)))
    assert moved, "the rewritten query must change the Top-K for the check to mean anything"
