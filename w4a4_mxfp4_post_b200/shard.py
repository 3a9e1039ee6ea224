"""Host-side partitioning of a batch across ranks (one process per GPU).

The quantizer is row-independent: every token row of X is quantized on its
own, so a batch splits across ranks by contiguous row ranges with no data
exchange, each rank holding a replica of the (small) factors.
"""


def row_range(M: int, world: int, rank: int) -> tuple:
    """Contiguous rows [r0, r1) of an M-row batch owned by `rank` of `world`.

    Ranges differ in size by at most one row and cover 0..M exactly once.
    """
    if world < 1 or not (0 <= rank < world) or M < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, M >= 0")
    base, extra = divmod(M, world)
    r0 = rank * base + min(rank, extra)
    r1 = r0 + base + (1 if rank < extra else 0)
    return r0, r1
