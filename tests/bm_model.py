"""A separately written Python model of the block manager's rules, for the tests.

Rules (from the pages: blocks on demand, freed at once, shared between sequences with
a reference count, a private copy before writing into a shared partially filled
block): allocate ceil(n / bs) blocks; fork shares every block; free returns blocks
whose count reaches 0; append reserves position L of each sequence.  Free blocks are
handed out last-returned-first, lowest id first at the start.
"""


class NoBlocks(Exception):
    pass


class Model:
    def __init__(self, num_blocks, block_size):
        self.bs = block_size
        self.ref = [0] * num_blocks
        self.free_ids = list(range(num_blocks))[::-1]
        self.seqs = {}  # id -> (blocks list, length)

    def _take(self):
        b = self.free_ids.pop()
        self.ref[b] = 1
        return b

    def _drop(self, b):
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free_ids.append(b)

    def allocate(self, sid, n):
        if sid in self.seqs:
            raise KeyError(sid)
        need = -(-n // self.bs)
        if need > len(self.free_ids):
            raise NoBlocks()
        self.seqs[sid] = ([self._take() for _ in range(need)], n)

    def fork(self, parent, child):
        if child in self.seqs or parent not in self.seqs:
            raise KeyError(child)
        blocks, n = self.seqs[parent]
        for b in blocks:
            self.ref[b] += 1
        self.seqs[child] = (list(blocks), n)

    def free(self, sid):
        blocks, _ = self.seqs.pop(sid)
        for b in reversed(blocks):
            self._drop(b)

    def append(self, ids):
        # count first: all or nothing
        held = {}
        need = 0
        for sid in ids:
            blocks, n = self.seqs[sid]
            if n % self.bs == 0:
                need += 1
            else:
                b = blocks[-1]
                if self.ref[b] - held.get(b, 0) > 1:
                    need += 1
                    held[b] = held.get(b, 0) + 1
        if need > len(self.free_ids):
            raise NoBlocks()
        slots, pairs = [], []
        for sid in ids:
            blocks, n = self.seqs[sid]
            off = n % self.bs
            if off == 0:
                b = self._take()
                blocks.append(b)
            else:
                b = blocks[-1]
                if self.ref[b] > 1:
                    c = self._take()
                    pairs.append((b, c))
                    self._drop(b)
                    blocks[-1] = c
                    b = c
            slots.append(b * self.bs + off)
            self.seqs[sid] = (blocks, n + 1)
        return slots, pairs
