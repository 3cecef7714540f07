"""The decode attention kernel's context split and stage schedule, checked on
the CPU for every chunks-per-CTA count F.

attn_decode_tc_kernel (weight_shared_looped_b200/csrc/attention.cu) splits a
lane's n_keys = pos + 1 keys into CL = min(8, ceil(max_ctx / 64)) chunks of
per = ceil(n_keys / CL) keys; CTA r of the cluster takes chunks r*F .. r*F+F-1
and streams them in 64-key stages, each chunk from its own start.  The stage
arithmetic below is the kernel's (stage s -> chunk j, keys [lo, lo + cnt) of
the CTA; a row is copied from the cache if it holds an older key, left to the
append if it is the new key, zero-filled otherwise).  The checks: every key is
read exactly once, by the chunk key // per whatever F is (so the fold order,
and with it every rounding, does not depend on F); the new key's row is never
copied and is appended by exactly one CTA in exactly one stage; each chunk's
end is detected at its last stage; the scale buffer covers every row read."""
import pytest

DS_KEYS = 64   # keys per stage
MAX_CHUNKS = 8


def cluster_size(max_ctx):
    return max(1, min(MAX_CHUNKS, (max_ctx + 63) // 64))


def scale_len(max_ctx, F):
    CL = cluster_size(max_ctx)
    max_per = (max_ctx + CL - 1) // CL
    return (F * max_per + DS_KEYS + 7) // 8 * 8


def stage_keys(s, NSF, per, nkc):
    j, sub = divmod(s, NSF)
    nkj = min(per, nkc - j * per)
    lo = j * per + sub * DS_KEYS
    cnt = min(DS_KEYS, nkj - sub * DS_KEYS)
    return lo, cnt, nkj, j


def check(max_ctx, pos, F, mode=0):
    """mode 0: the CTA holding key pos appends it (the decode step); mode 2:
    every key, pos included, is copied from the cache (the attend pass after
    an append pass)."""
    CL = cluster_size(max_ctx)
    n_keys = pos + 1
    per = (n_keys + CL - 1) // CL
    sc_len = scale_len(max_ctx, F)
    ctas = (CL + F - 1) // F
    reads = [0] * n_keys
    appends = 0
    for crank in range(ctas):
        kA = min(crank * F * per, n_keys)
        kB = min(kA + F * per, n_keys)
        nkc = kB - kA
        owner = mode != 2 and nkc > 0 and kB == n_keys
        n_old = nkc - 1 if owner else nkc
        NSF = (per + DS_KEYS - 1) // DS_KEYS
        nstage = nkc // per * NSF + (nkc % per + DS_KEYS - 1) // DS_KEYS
        ends = []
        for s in range(nstage):
            lo, cnt, nkj, j = stage_keys(s, NSF, per, nkc)
            assert 1 <= cnt <= DS_KEYS and j < F
            chunk = crank * F + j
            assert chunk < CL
            rnew = n_old - lo if owner and n_old - lo < cnt else -DS_KEYS
            rem = min(cnt, n_old - lo)
            # the stage into which the main loop writes the appended entry
            inject = owner and lo <= n_old < lo + cnt
            assert inject == (rnew >= 0)
            for r in range(DS_KEYS):
                key = kA + lo + r
                if r == rnew:                     # left to the append
                    assert key == pos
                    appends += 1
                elif r < rem:                     # copied from the cache
                    assert key < pos or (mode == 2 and key == pos)
                else:                             # zero-filled (past the stage's keys)
                    assert r >= cnt
                if r < cnt:
                    reads[key] += 1
                    assert key // per == chunk    # the chunk the fixed split puts it in
                assert lo + r < sc_len            # scale of every row the lanes read
            # the kernel closes a chunk when the stage reaches the chunk's last key
            if lo + cnt - j * per == nkj:
                ends.append(j)
        assert ends == [j for j in range(F) if min(per, nkc - j * per) > 0]
    assert reads == [1] * n_keys
    assert appends == (1 if mode == 0 else 0)


CTX = [1, 2, 16, 63, 64, 65, 100, 128, 200, 384, 511, 512, 513, 1056, 2048, 2112, 4096, 5000]


@pytest.mark.parametrize("max_ctx", CTX)
def test_stage_schedule_covers_each_key_once_for_every_F(max_ctx):
    positions = {0, 1, 2, 63, 64, 65, 127, 128, 255, 256, 257,
                 max_ctx // 3, max_ctx // 2, max_ctx - 2, max_ctx - 1}
    for pos in sorted(p for p in positions if 0 <= p < max_ctx):
        for F in range(1, cluster_size(max_ctx) + 1):
            check(max_ctx, pos, F)
            check(max_ctx, pos, F, mode=2)


def test_chunk_count_follows_the_cache_size():
    assert [cluster_size(c) for c in (1, 64, 65, 128, 448, 449, 512, 4096)] == \
        [1, 1, 2, 2, 7, 8, 8, 8]


def test_model_follows_the_kernel_source():
    """The arithmetic modelled above is the kernel's, line for line; a change
    there must be carried into the model."""
    import os
    import re
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with open(os.path.join(root, "weight_shared_looped_b200", "csrc", "attention.cu")) as f:
        src = re.sub(r"\s+", " ", f.read())
    for line in [
        "constexpr int DS_KEYS = 64;",
        "const int c = (max_ctx + 63) / 64;",
        "const int per = (n_keys + CL - 1) / CL;",
        "const int kA = min(crank * F * per, n_keys), kB = min(kA + F * per, n_keys);",
        "const bool owner = a.mode != 2 && nkc > 0 && kB == n_keys;",
        "const int pos = a.hdr->pos[lane_id] + a.row_off[row];",
        "const int n_old = owner ? nkc - 1 : nkc;",
        "const int NSF = (per + DS_KEYS - 1) / DS_KEYS;",
        "const int nstage = nkc / per * NSF + (nkc % per + DS_KEYS - 1) / DS_KEYS;",
        "nkj = min(per, nkc - j * per);",
        "lo = j * per + sub * DS_KEYS;",
        "cnt = min(DS_KEYS, nkj - sub * DS_KEYS);",
        "const int rnew = owner && n_old - lo < cnt ? n_old - lo - cr0 : -DS_KEYS;",
        "const int rem = min(cnt, n_old - lo) - cr0;",
        "if (base + cnt - jc * per == nkj)",
        "if (owner && n_old >= base && n_old - base < cnt && tid < HD)",
        "const int max_per = (a.max_ctx + cl - 1) / cl;",
        "(f * max_per + DS_KEYS + 7) / 8 * 8",
    ]:
        assert line in src, line
