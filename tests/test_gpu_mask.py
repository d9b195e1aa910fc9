"""Bit-exact masks: the CUDA path attends exactly the oracle's visible sets.

With q = 0 every score is 0 (QK-norm maps 0 to 0), so each row's softmax is
uniform over its visible set:
  * exp(lse_i) = |A(i)| exactly (the count is recovered by rounding);
  * with v one-hot in channel d at a probe key j_d, out[i, d] is 1/|A(i)|
    when j_d is visible from i and exactly 0 when it is not.
Each (kv head, channel) probes its own key, so one call checks membership of
Hkv * D keys for every row; probes sit at tile, window and span edges.
"""
import numpy as np
import pytest
import torch

import global_gqa_b200 as g3
import inputs
from oracle import attention as O
from gpu_helpers import dev, to_dev

pytestmark = pytest.mark.gpu


def _probe_keys(S, W, spans_b, n, rng):
    cand = set()
    for e in list(range(0, S, 128)) + [W - 1, W, W + 1, S - 1, S - 2]:
        for d in (-2, -1, 0, 1):
            if 0 <= e + d < S:
                cand.add(e + d)
    if spans_b is not None:
        for st, en in np.asarray(spans_b).reshape(-1, 2):
            for e in (st - 1, st, st + 1, en - 2, en - 1, en):
                if 0 <= e < S:
                    cand.add(int(e))
    cand = sorted(cand)
    rng.shuffle(cand)
    extra = rng.integers(0, S, n).tolist()
    keys = (cand + extra)[:n]
    while len(keys) < n:
        keys.append(int(rng.integers(0, S)))
    return np.array(keys)


CASES = [
    # B, S, Hq, Hkv, D, kind, W, spans
    (1, 2048, 4, 2, 64, O.LOCAL, 1024, None),
    (1, 2048, 4, 2, 64, O.GLOBAL, 1024, None),
    (2, 1500, 4, 2, 128, O.LOCAL, 300, [[0, 256], [256, 512], [900, 1156]]),
    (1, 4000, 4, 2, 128, O.LOCAL, 1024, [[1, 2], [1500, 3100]]),
    (1, 999, 2, 2, 64, O.GLOBAL, 1, [[300, 556], [998, 999]]),
    (2, 32768, 32, 16, 128, O.LOCAL, 1024, "mixed"),
    (2, 32768, 32, 16, 128, O.GLOBAL, 1024, "mixed"),
]


@pytest.mark.parametrize("case", CASES, ids=[f"S{c[1]}_k{c[5]}_W{c[6]}_{'sp' if c[7] else 'nosp'}" for c in CASES])
def test_visible_sets_exact(case):
    B, S, Hq, Hkv, D, kind, W, spans = case
    rng = np.random.default_rng(S + W + kind)
    if spans == "mixed":
        sp = inputs.image_spans(B, S, 8, seed=0)
    elif spans is None:
        sp = None
    else:
        sp = torch.tensor([spans] * B, dtype=torch.int32)
    x = inputs.prefill_layer_inputs(B, S, Hq, Hkv, D, seed=11)
    x["q"] = torch.zeros_like(x["q"])
    probes = np.zeros((B, Hkv, D), dtype=np.int64)
    v = torch.zeros(B, S, Hkv, D, dtype=torch.bfloat16)
    for b in range(B):
        for h in range(Hkv):
            keys = _probe_keys(S, W, None if sp is None else sp[b].numpy(), D, rng)
            probes[b, h] = keys
            v[b, keys, h, np.arange(D)] = 1.0
    x["v"] = v
    x["spans"] = sp
    xd = to_dev(x)
    out, lse = g3.prefill(xd["q"], xd["k"], xd["v"], xd["q_gamma"], xd["k_gamma"], xd["positions"], kind, W,
                          1e4, 1.0, xd["spans"], return_lse=True)
    assert g3.check_device_error(g3.workspace(0, dev())) == 0
    outc = out.float().cpu().numpy()
    cnt = np.rint(np.exp(lse.double().cpu().numpy())).astype(np.int64)   # [B, Hq, S]
    G = Hq // Hkv
    for b in range(B):
        sid = O.span_ids(S, None if sp is None else sp[b].numpy())
        rows = np.arange(S)
        # counts for every row and head
        want = np.array([np.count_nonzero(O.allowed_row(i, S, kind, W, sid)) for i in rows])
        assert (cnt[b] == want[None, :]).all(), "visible-set sizes differ"
        # membership of every probe key for every row
        for h in range(Hq):
            kv = h // G
            vis = O.allowed(rows[:, None], probes[b, kv][None, :], kind, W, sid)       # [S, D]
            got = outc[b, :, h, :] != 0
            assert np.array_equal(got, vis), f"membership differs (b={b}, head={h})"
