"""Head sharding of one layer across ranks (one process per GPU).

Every (b, h) plane of the layer is an independent problem: its own k-means, selection, permutation
and attention (the pages' Method (1)-(4) act per head).  So G ranks can take H/G heads each with no
exchange on the data path; each rank calls the library on its contiguous block of heads, and the
outputs stay sharded by head (as a head-parallel model keeps them until its output projection).
"""


def head_range(H: int, world: int, rank: int):
    """Contiguous block [h0, h1) of the H heads for `rank` of `world`: sizes differ by at most one,
    the first H % world ranks taking the extra head.  Ranks past H get an empty block."""
    if H < 0 or world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad shard: H={H} world={world} rank={rank}")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)
