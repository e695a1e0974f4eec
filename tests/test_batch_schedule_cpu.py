"""The persistent batch kernel's work split, checked on the CPU for many shapes.

Rules (as documented in the kernel): stages are numbered item-major, then row-block-major, then
along K; CTA c owns [c T / G, (c + 1) T / G).  A row block whose stages fall to several CTAs is
summed through the workspace: contributor c stores its partial in slot 2c if the block holds the
first stage of c's range, else in slot 2c + 1; the arrivals are counted on counter[first
contributor]; the last contributor reads the slots of the first..last contributor.  These checks
make sure no two partials share a slot, no two split blocks share a counter, every contributor
is found by the reader, and every stage is owned by exactly one CTA."""
import random


def range_begin(c, T, G):
    return c * T // G


def owner(s, T, G):
    return ((s + 1) * G - 1) // T


def check(blocks, G):
    """blocks: list of stage counts per row block (items concatenated)."""
    T = sum(blocks)
    G = min(G, T)
    begin = 0
    slot_owner = {}
    counters = {}
    for C in blocks:
        b0, b1 = begin, begin + C
        begin = b1
        cf, cl = owner(b0, T, G), owner(b1 - 1, T, G)
        # the contributors are exactly the CTAs whose ranges intersect [b0, b1)
        inter = [c for c in range(G) if max(range_begin(c, T, G), b0) < min(range_begin(c + 1, T, G), b1)]
        assert inter == list(range(cf, cl + 1))
        if cf == cl:
            s0, s1 = range_begin(cf, T, G), range_begin(cf + 1, T, G)
            assert b0 >= s0 and b1 <= s1          # whole: finished in one CTA
            continue
        assert cf not in counters
        counters[cf] = (b0, b1)
        for c in range(cf, cl + 1):
            s0 = range_begin(c, T, G)
            writer_slot = 2 * c + (0 if b0 <= s0 else 1)
            reader_slot = 2 * c + (0 if b0 <= range_begin(c, T, G) else 1)
            assert writer_slot == reader_slot
            assert writer_slot not in slot_owner, (writer_slot, slot_owner[writer_slot], (b0, b1))
            slot_owner[writer_slot] = (b0, b1)
    # every stage has exactly one owner
    for s in range(T):
        c = owner(s, T, G)
        assert range_begin(c, T, G) <= s < range_begin(c + 1, T, G)


def test_llama_and_qwen_layers():
    llama = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096), (14336, 4096), (4096, 14336)]
    qwen = [(4608, 3584), (3584, 3584), (37888, 3584), (3584, 18944)]
    for shapes in (llama, qwen):
        for stage_k in (512, 256):                     # ternary, W4A16
            blocks = []
            for N, K in shapes:
                blocks += [-(-K // stage_k)] * (-(-N // 128))
            for G in (2 * 148, 2 * 132, 2 * 114, 7, 1):
                check(blocks, G)


def test_random_shapes():
    rng = random.Random(0)
    for _ in range(400):
        blocks = []
        for _ in range(rng.randint(1, 8)):
            blocks += [rng.randint(1, 40)] * rng.randint(1, 60)
        check(blocks, rng.randint(1, 400))
