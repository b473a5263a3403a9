"""Host-side bound of the decode attention's split-K records (no GPU needed).

The attention streams 32-key tiles in two phases, every unit's window then compressed-token
tiles (phase A) and then every unit's selected-block tiles (phase B), each phase cut into equal
contiguous ranges, one per warp (SM count x 4 warps wanted). A warp writes one record per
(unit, branch) piece it covers, into slot `warp - first warp of that piece`. The library sizes
the workspace for these slots; this test walks every warp of the partition for a spread of
shapes and checks that the workspace the library asks for holds every slot written."""
import random

import pytest

from block_sparse_long_summary_b200 import build as B

TK = 32          # keys per tile
SMS = 148        # the library's SM count when no device is present
WARPS = 4        # warps per attention CTA


@pytest.fixture(scope="module")
def lib():
    B.build()
    from block_sparse_long_summary_b200 import cobs
    return cobs


def slots_needed(units, tS, tW, tC):
    """Largest slot index + 1 any (unit, branch) piece uses, walking every warp's ranges."""
    tAu = tW + tC
    nA, nBt = units * tAu, units * tS
    want = SMS * WARPS
    tpwA, tpwB = max(1, -(-nA // want)), max(1, -(-nBt // want))
    nw = max(-(-nA // tpwA), -(-nBt // tpwB))
    first = {}
    need = 0
    for v in range(nw):
        pieces = []
        for g in range(v * tpwA, min(nA, v * tpwA + tpwA)):
            u, l = divmod(g, tAu)
            pieces.append((u, 1 if l < tW else 2, (u * tAu + (0 if l < tW else tW)) // tpwA))
        for g in range(v * tpwB, min(nBt, v * tpwB + tpwB)):
            u = g // tS
            pieces.append((u, 0, (u * tS) // tpwB))
        for u, br, fv in set(pieces):
            first.setdefault((u, br), fv)
            need = max(need, v - fv + 1)
    return need


SHAPES = [
    dict(B=8, Hq=32, Hkv=8, d=128, T=32768, topk=16, window=512),    # 32k decode workload
    dict(B=1, Hq=64, Hkv=8, d=128, T=131072, topk=32, window=1024),  # 128k decode workload
    dict(B=1, Hq=4, Hkv=4, d=128, T=65536, topk=16, window=512),
    dict(B=2, Hq=4, Hkv=2, d=64, T=4096 + 37, topk=16, window=512),
    dict(B=3, Hq=2, Hkv=2, d=64, T=1000, topk=4, window=128),
    dict(B=1, Hq=1, Hkv=1, d=64, T=100, topk=1, window=64),
]
rng = random.Random(7)
for _ in range(12):
    hkv = rng.choice([1, 2, 4, 8])
    SHAPES.append(dict(B=rng.randint(1, 40), Hq=hkv * rng.choice([1, 2, 4]), Hkv=hkv, d=rng.choice([64, 128]),
                       T=rng.randint(64, 300000), topk=rng.randint(1, 32), window=rng.choice([64, 512, 1024])))


@pytest.mark.parametrize("shape", SHAPES)
def test_workspace_holds_every_record_slot(lib, shape):
    p = lib.Params(dtype="bf16", **shape)
    units, G = shape["B"] * shape["Hkv"], shape["Hq"] // shape["Hkv"]
    tS = shape["topk"] * (64 // TK)
    tW = -(-min(shape["window"], shape["T"]) // TK)
    nC = 0 if shape["T"] < 32 else (shape["T"] - 32) // 16 + 1
    tC = -(-nC // TK)
    need = slots_needed(units, tS, tW, tC)
    rec_bytes = G * (shape["d"] + 4) * 4
    ws = lib.workspace_bytes(p, lib.COBS_WS_DECODE)
    assert ws >= units * 3 * need * rec_bytes, (ws, need)
