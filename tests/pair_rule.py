"""The query-block pairing rule stated plainly in Python, for the tests.

Pairing only decides which two query blocks share a 128-row attention tile; it never
changes a result.  The GPU pass (sba_pair_query_blocks) must give exactly this tile list
for the routing it is handed."""
import numpy as np


def host_pairing(idx, cnt, nB, nQ, window=64, n_cands=16, rounds=4):
    """The pairing rule of one (b, h), stated plainly: each valid query block that does not
    keep every block ranks the valid blocks within +-window positions by kept-set overlap,
    then nearness, then the lower index, and keeps its n_cands best; in round 0 it proposes
    its best, in later rounds its first candidate still unmatched; mutual proposals match.
    Tiles: matched pairs by their lower block, then the unmatched valid blocks in order,
    then the blocks past the valid length, two by two, -1 filling an odd count."""
    kmax = idx.shape[1]
    bits = np.zeros((nQ, nQ), dtype=np.int64)
    for a in range(nQ):
        c = min(max(int(cnt[a]), 0), kmax)
        J = idx[a, :c]
        bits[a, J[(J >= 0) & (J < nQ)]] = 1
    ov = bits @ bits.T
    cands = [[] for _ in range(nQ)]
    for a in range(nB):
        if cnt[a] >= nB:
            continue
        keys = [(int(ov[a, c]), -abs(c - a), 1 if c < a else 0, c)
                for c in range(max(0, a - window), min(nB, a + window + 1)) if c != a]
        keys.sort(reverse=True)
        cands[a] = [kk[3] for kk in keys[:n_cands]]
    partner = np.full(nQ, -1)
    prop = np.array([cs[0] if cs else -1 for cs in cands])
    for r in range(rounds):
        if r > 0:
            prop = np.full(nQ, -1)
            for a in range(nQ):
                if partner[a] < 0:
                    for c in cands[a]:
                        if partner[c] < 0:
                            prop[a] = c
                            break
        for a in range(nQ):
            c = prop[a]
            if c >= 0 and partner[a] < 0 and prop[c] == a:
                partner[a] = c
    order = []
    for a in range(nB):
        if partner[a] > a:
            order += [a, int(partner[a])]
    order += [a for a in range(nB) if partner[a] < 0]
    order += list(range(nB, nQ))
    order += [-1] * (2 * ((nQ + 1) // 2) - len(order))
    return np.array(order, dtype=np.int32)
