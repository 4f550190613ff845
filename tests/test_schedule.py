"""Host tile scheduler (CPU): tile classes against brute force over a dense
mask, pair counts against closed forms, and the work list's coverage and
longest-first order."""
import numpy as np
import pytest

import attention_jvp_continuous_b200 as ja
from attention_jvp_continuous_b200 import build
from oracle import MaskSpec, key_intervals


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def dense(spec):
    L = spec.length
    m = np.zeros((L, L), dtype=bool)
    for i in range(L):
        for a, b in key_intervals(spec, i):
            m[i, a:b] = True
    return m


def brute_classes(m, bm, bn):
    L = m.shape[0]
    nq, nk = -(-L // bm), -(-L // bn)
    out = np.zeros((nq, nk), dtype=np.int8)
    for qt in range(nq):
        for kt in range(nk):
            blk = m[qt * bm:(qt + 1) * bm, kt * bn:(kt + 1) * bn]
            ragged = (kt + 1) * bn > L
            if not blk.any():
                out[qt, kt] = 0
            elif blk.all() and not ragged:
                out[qt, kt] = 1
            else:
                out[qt, kt] = 2
    return out


CASES = []
rng = np.random.default_rng(0)
for n in range(24):
    mode = n % 4
    CASES.append((mode, int(rng.integers(1, 40)), int(rng.integers(1, 9)),
                  int(rng.integers(1, 4)), int(rng.choice([8, 16, 32, 128])),
                  int(rng.choice([8, 16, 64]))))


# The backward's query pass runs 128 x 128 tiles: ragged lengths, lengths
# below one tile, and each mask mode.
QCASES = [(ja.TEACHER_FORCING, 200, 3, 1, 128, 128), (ja.TEACHER_FORCING, 100, 5, 2, 128, 128),
          (ja.FRAME_CAUSAL, 130, 5, 1, 128, 128), (ja.CHUNK_CAUSAL, 70, 7, 3, 128, 128),
          (ja.DENSE, 64, 4, 1, 128, 128), (ja.TEACHER_FORCING, 5, 2, 1, 128, 128)]


@pytest.mark.parametrize("mode,T,F,ch,bm,bn", CASES + QCASES)
def test_tile_classes_match_brute_force(mode, T, F, ch, bm, bn):
    spec = MaskSpec(mode, T, F, ch)
    got = ja.tile_classes(ja.Mask(mode, T, F, ch), bm=bm, bn=bn)
    want = brute_classes(dense(spec), bm, bn)
    np.testing.assert_array_equal(got, want)
    pairs, full, partial, empty = ja.mask_stats(ja.Mask(mode, T, F, ch), bm=bm, bn=bn)
    assert pairs == int(dense(spec).sum())
    assert (full, partial, empty) == tuple(int((want == c).sum()) for c in (1, 2, 0))


@pytest.mark.parametrize("mode,T,F,ch,bm,bn", CASES[:12] + QCASES)
def test_schedule_covers_nonempty_tiles_in_order(mode, T, F, ch, bm, bn):
    mk = ja.Mask(mode, T, F, ch)
    cls = ja.tile_classes(mk, bm=bm, bn=bn)
    qt, sg = ja.schedule(mk, bm=bm, bn=bn)
    assert sorted(qt[:, 0].tolist()) == list(range(cls.shape[0]))
    # longest first
    assert np.all(np.diff(qt[:, 3]) <= 0)
    for q, s0, sc, nkt in qt:
        seen = np.zeros(cls.shape[1], dtype=np.int8)
        prev_end = -1
        for kb, cnt, part in sg[s0:s0 + sc]:
            assert kb >= prev_end and cnt >= 1
            prev_end = kb + cnt
            seen[kb:kb + cnt] = 2 if part else 1
        np.testing.assert_array_equal(seen, cls[q])
        assert nkt == int((cls[q] > 0).sum())


def test_workload_pair_counts_and_tile_tables():
    T = 1560
    assert ja.mask_stats(ja.Mask(ja.FRAME_CAUSAL, T, 21))[0] == 562_161_600
    assert ja.mask_stats(ja.Mask(ja.TEACHER_FORCING, T, 21, 1))[0] == 1_124_323_200
    assert ja.mask_stats(ja.Mask(ja.TEACHER_FORCING, T, 21, 3))[0] == 1_226_534_400
    assert ja.mask_stats(ja.Mask(ja.TEACHER_FORCING, T, 33, 1))[0] == 2_730_499_200
    # 128 x 128 tiling of the 65,520-token teacher-forcing mask. Query rows
    # past L are never written, so the ragged last query tile can be FULL.
    p, full, part, empty = ja.mask_stats(ja.Mask(ja.TEACHER_FORCING, T, 21, 1), bm=128, bn=128)
    assert (full, part) == (67_487, 2_133)
    assert full + part + empty == 512 * 512
    # the 128 x 64 grid the tensor-core kernel runs
    p64, full64, part64, _ = ja.mask_stats(ja.Mask(ja.TEACHER_FORCING, T, 21, 1))
    assert (full64, part64) == (135_469, 3_259)
    # admitted slots in visited tiles bound the pair count
    assert full * 128 * 128 <= p <= (full + part) * 128 * 128


def test_every_query_tile_has_work():
    for mk in (ja.Mask(ja.TEACHER_FORCING, 1560, 21, 1), ja.Mask(ja.FRAME_CAUSAL, 7, 5),
               ja.Mask(ja.TEACHER_FORCING, 3, 4, 3), ja.Mask(ja.DENSE, 5, 5)):
        qt, _ = ja.schedule(mk)
        assert np.all(qt[:, 3] >= 1)


def test_schedule_rejects_bad_descriptor():
    with pytest.raises(ja.JvpAttnError):
        ja.mask_stats(ja.Mask(ja.TEACHER_FORCING, 4, 4, 1), L=33)


@pytest.mark.parametrize("mode,T,F,ch,bm,bn", CASES[:12])
def test_key_pass_schedule_is_the_transposed_grid(mode, T, F, ch, bm, bn):
    # key tiles of bk = bm keys, query tiles of bq = bn rows
    mk = ja.Mask(mode, T, F, ch)
    L = mk.length
    cls = brute_classes(dense(MaskSpec(mode, T, F, ch)), bn, bm)  # [query tile, key tile]
    nq = cls.shape[0]
    for qt in range(nq):  # query rows past L must be masked in this pass
        if (qt + 1) * bn > L:
            cls[qt][cls[qt] == 1] = 2
    kt_list, sg = ja.schedule_kv(mk, bq=bn, bk=bm)
    assert np.all(np.diff(kt_list[:, 3]) <= 0)
    covered = set()
    for kt, s0, sc, nqt in kt_list:
        seen = np.zeros(nq, dtype=np.int8)
        for qb, cnt, part in sg[s0:s0 + sc]:
            seen[qb:qb + cnt] = 2 if part else 1
        np.testing.assert_array_equal(seen, cls[:, kt])
        assert nqt == int((cls[:, kt] > 0).sum())
        covered.add(int(kt))
    # every key tile with an admitted pair has an entry
    assert covered == {kt for kt in range(cls.shape[1]) if (cls[:, kt] > 0).any()}
