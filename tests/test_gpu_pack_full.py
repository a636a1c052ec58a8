"""Packing is bit-exact at full size, on the weights of every workload.

The 2:4 selection of the sparse region (SpenseGPT page, Technical Summary §1:
two of every four consecutive weights are zero; ties to the lower index) and
the split into the 2:4 region and the dense region (§2.A, with §2.B's tail or
scattered dense set) must give exactly the bytes the oracle gives. Each
workload's weights are packed at their full shape: the 32B attention
projections, the 32B FFN with its x20 weight outliers, the SpenseGPT+ down
projection at every dense fraction of its sweep (scattered dense sets), and
the six weights of the 36B layer. The packed arrays (MMA-tiled and canonical)
are compared byte for byte with the oracle's pack and tiling of the same rows
on the first, the last and 16 random 128-row tiles (every tile of a weight of
at most 32 tiles).

The weights are drawn on the GPU by the seeded input generator (synth), the
way the benchmark draws them, and copied to the host for the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from dense_fp8_gemm_b200 import spense, synth, workloads

pytestmark = pytest.mark.gpu

CASES = []
for _wl in (workloads.ATTN32B, workloads.FFN32B, workloads.CHAIN36B):
    for _i, (_label, _N, _K) in enumerate(_wl.shapes):
        CASES.append((_wl.name, _i, 0.25))
for _df in workloads.SPENSE_PLUS.dense_fracs:
    CASES.append((workloads.SPENSE_PLUS.name, 0, _df))


def sampled_tiles(n_tiles, seed):
    if n_tiles <= 32:
        return np.arange(n_tiles)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, n_tiles - 1), 16, replace=False)
    return np.concatenate([[0], np.sort(mid), [n_tiles - 1]])


@pytest.mark.parametrize("wl_name,i,df", CASES, ids=[f"{w}-{i}-df{d}" for w, i, d in CASES])
def test_full_size_pack_bit_exact(wl_name, i, df):
    wl = workloads.BY_NAME[wl_name]
    label, N, K = wl.shapes[i]
    Kd = workloads.dense_count(K, df)
    Ks = K - Kd
    idx = synth.scored_dense_idx(wl.seed, 102 + 10 * i, K, Kd) if wl.scattered else None
    q, s = synth.device_fp8_rows(wl.seed, workloads.weight_id(i), (N, K), wl.w_std, "cuda",
                                 outliers=wl.outliers)
    pw = spense.pack(q, s, Kd=Kd, dense_idx=idx, keep_canonical=True)
    torch.cuda.synchronize()
    n_tiles = (N + 127) // 128
    tiles = sampled_tiles(n_tiles, N + K + Kd)
    rows = np.concatenate([np.arange(t * 128, min(N, (t + 1) * 128)) for t in tiles])
    W = q[torch.from_numpy(rows).cuda()].cpu().numpy()
    del q
    ref = oracle.pack(W, dense_idx=idx, Kd=Kd)
    tref = oracle.tile(ref["Vs"], ref["E"], ref["Wd"], rows.size, Ks, Kd)
    nsb, ndb = -(-Ks // 256), -(-Kd // 128)
    for name, per_tile in (("Vs_t", nsb * 16384), ("E_t", nsb * 4096), ("Wd_t", ndb * 16384)):
        if per_tile == 0:
            assert pw.view(name) is None
            continue
        full = pw.view(name).view(n_tiles, per_tile)
        got = full[torch.from_numpy(tiles).cuda()].cpu().numpy().reshape(-1)
        np.testing.assert_array_equal(got, tref[name], err_msg=f"{label} {name}")
    sel = torch.from_numpy(rows).cuda()
    for name in ("Vs", "E", "Wd"):
        v = pw.view(name)
        got = np.zeros(ref[name].shape, np.uint8) if v is None else v[sel].cpu().numpy()
        np.testing.assert_array_equal(got, ref[name], err_msg=f"{label} {name}")
    np.testing.assert_array_equal(pw.view("w_scale")[sel].cpu().numpy(), s[sel].cpu().numpy())
    pw.free()
