"""The full-size parity tests compare a token sample chosen so that every
tile of the grouped GEMMs has rows compared; this checks that choice on the
CPU against a brute-force walk of the CSR."""
import numpy as np
import pytest

import oracle
from gpu_helpers import every_tile_tokens


@pytest.mark.parametrize("T,E,k,seed,mask_frac", [(4096, 8, 2, 0, 0.0), (2048, 128, 4, 1, 0.0), (300, 16, 6, 2, 0.3),
                                                  (5000, 8, 2, 3, 0.3)])
def test_every_piece_of_every_expert_is_sampled(T, E, k, seed, mask_frac):
    rng = np.random.default_rng(seed)
    idx = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    mask = (rng.random(T) >= mask_frac).astype(np.uint8) if mask_frac > 0 else None
    tokens = set(every_tile_tokens(idx, E, token_mask=mask).tolist())
    # the CSR of the live slots, from the oracle's counting sort
    live = idx.copy()
    if mask is not None:
        live = idx[mask != 0]
        tok_of = np.flatnonzero(mask != 0)
    else:
        tok_of = np.arange(T)
    _, off, perm, _ = oracle.create_indices(live, E)
    for e in range(E):
        lo, hi = off[e], off[e + 1]
        for p0 in range(lo, hi, 128):
            p1 = min(p0 + 128, hi)
            owners = {int(tok_of[s // k]) for s in perm[p0:p1]}
            assert owners & tokens, (e, p0)
            if p1 == hi:
                assert owners <= tokens, (e, p0)
    if mask is not None:
        assert not (tokens & set(np.flatnonzero(mask == 0).tolist()))
    assert len(tokens) <= T
