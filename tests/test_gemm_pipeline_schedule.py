"""Host replay of the fused GEMM's dequantizing schedule (csrc/nf4_gemm.cu).

One CTA per tile: 16 dequantizing warps, one group, 3 w_hat tiles (register sets).  A CTA
pair: 4 groups of 4 warps taking the steps in turn over 4 half-size w_hat tiles, one
register set each.  Group g's loop visits i0 = 0, S, 2S, .. and, for register set v, the
step i = i0 + v G + g on tile u = v G + g (S tiles, G groups); it prefetches step i + S into
the set it has just used.  This replays that loop for every step count and checks that:
- each step is dequantized exactly once, on tile i mod S, from inputs fetched for it;
- the arrivals on each tile's "full" barrier per phase equal its initial count (every thread
  of the group per step, or one per warp of the group in each of the pair's CTAs);
- the parity a step waits on for its tile's "empty" barrier is the phase of the step that
  last used the tile.
"""
import pytest

DEQ_WARPS = 16


def replay(nk, pair):
    S = 4 if pair else 3            # w_hat tiles
    G = 4 if pair else 1            # groups
    sets = S // G
    assert sets * G == S
    full_count = 2 * DEQ_WARPS // G if pair else 32 * DEQ_WARPS
    arrivals = {}                   # (tile, phase) -> arrivals on the full barrier
    done = {}
    for g in range(G):
        fetched = {v: v * G + g for v in range(sets)}  # register set -> step it holds
        going, i0 = True, 0
        while i0 < nk and going:
            for v in range(sets):
                u = v * G + g
                i = i0 + u
                if not going:
                    continue
                if i >= nk:
                    going = False
                    continue
                assert fetched[v] == i, "the set holds this step's codes"
                assert u == i % S
                if i >= S:  # waits on the empty barrier of tile u for the step S before
                    parity = (i // S - 1) & 1
                    assert parity == ((i - S) // S) & 1
                assert i not in done
                done[i] = g
                warps = DEQ_WARPS // G
                per_step = 2 * warps if pair else 32 * warps  # per warp in each CTA / per thread
                arrivals[(u, i // S)] = arrivals.get((u, i // S), 0) + per_step
                fetched[v] = i + S
            i0 += S
    assert sorted(done) == list(range(nk))
    for (u, ph), n in arrivals.items():
        assert n == full_count, (u, ph, n)


@pytest.mark.parametrize("pair", [False, True])
@pytest.mark.parametrize("nk", list(range(1, 26)) + [64, 127, 128])
def test_each_step_dequantized_once_and_barrier_counts_match(nk, pair):
    replay(nk, pair)
