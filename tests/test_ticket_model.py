"""Host model of how the throughput-shape query kernel hands queries to its warps: every CTA
keeps a ticket counter in shared memory, its warps start with tickets 0 .. NW-1 and then take
the next ticket, and ticket t of CTA c is query (c + t // NW * grid) * NW + t % NW. A warp stops
at its first ticket whose query lies past the end. The model checks that, for any order in
which the warps take tickets, every query of the launch is handed out exactly once, and that the
tickets stay far below 2^31. It tests the scheme the CUDA code follows (query_kernels.cu,
query_kernel); the GPU parity tests check the code."""
import random

import pytest

NW = 14  # warps per CTA of the throughput shape


def query_of(c: int, t: int, grid: int) -> int:
    return (c + (t // NW) * grid) * NW + t % NW


def grid_for(num_queries: int, sms: int = 148, per_sm: int = 2) -> int:
    """The launcher's persistent grid: the resident CTAs, capped by the work."""
    need = (num_queries + NW - 1) // NW
    return min(need, sms * per_sm)


def run_cta(c: int, grid: int, num_queries: int, rng: random.Random):
    """Queries one CTA processes, its warps taking tickets in a random interleaving."""
    counter = NW
    current = {w: w for w in range(NW)}  # each warp's ticket
    done, last_ticket = [], 0
    while current:
        w = rng.choice(sorted(current))
        t = current[w]
        last_ticket = max(last_ticket, t)
        q = query_of(c, t, grid)
        if q >= num_queries:
            del current[w]  # the warp ends
            continue
        done.append(q)
        current[w] = counter  # the next ticket of this CTA
        counter += 1
    return done, last_ticket


@pytest.mark.parametrize("num_queries", [1, 13, 14, 15, 64, 1000, 4143, 4144, 4145, 65536,
                                         262144])
def test_every_query_once(num_queries):
    rng = random.Random(num_queries)
    grid = grid_for(num_queries)
    seen = []
    for c in range(grid):
        done, last = run_cta(c, grid, num_queries, rng)
        seen += done
        assert last < num_queries // grid + 2 * NW + NW  # far below 2^31
    assert sorted(seen) == list(range(num_queries))


@pytest.mark.parametrize("grid", [1, 2, 3, 7, 296])
def test_any_grid(grid):
    rng = random.Random(grid)
    num_queries = 3 * NW * grid + 5  # a ragged last chunk
    seen = []
    for c in range(grid):
        seen += run_cta(c, grid, num_queries, rng)[0]
    assert sorted(seen) == list(range(num_queries))


def test_neighbouring_queries_per_cta():
    """A CTA's first NW tickets are NW neighbouring queries (they share tree rows in L1)."""
    grid = 296
    for c in (0, 5, 295):
        qs = [query_of(c, t, grid) for t in range(NW)]
        assert qs == list(range(c * NW, c * NW + NW))
