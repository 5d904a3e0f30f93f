"""A separately written Python model of the block manager's rules, for the tests.

Rules (from the pages: blocks on demand, freed at once, shared between sequences with
a reference count, a private copy before writing into a shared partially filled
block): allocate ceil(n / bs) blocks; fork shares every block; free returns blocks
whose count reaches 0; append reserves position L of each sequence.  Free blocks are
handed out last-returned-first, lowest id first at the start.

Sliding window W (the blog's sliding_window setting, read as: a sequence of length L
needs only positions L-W .. L-1): a block whose positions all lie before L-W is given
back and its table entry becomes None.  A new sequence takes the blocks of all its
tokens (the prompt is attended in full); after an append batch the sequences of the
batch give back what fell out of their window.
"""


class NoBlocks(Exception):
    pass


class Model:
    def __init__(self, num_blocks, block_size, num_cpu_blocks=0, window=0):
        self.bs = block_size
        self.window = window
        self.ref = [0] * num_blocks
        self.free_ids = list(range(num_blocks))[::-1]
        self.seqs = {}  # id -> (blocks list, length)
        self.cpu_ref = [0] * num_cpu_blocks
        self.cpu_free = list(range(num_cpu_blocks))[::-1]
        self.on_cpu = set()

    def _take(self):
        b = self.free_ids.pop()
        self.ref[b] = 1
        return b

    def _drop(self, b):
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free_ids.append(b)

    def _dead(self, n):
        """Pages of a length-n context whose every position is before the window."""
        if self.window <= 0 or n <= self.window:
            return 0
        return sum(1 for j in range(-(-n // self.bs)) if (j + 1) * self.bs <= n - self.window)

    def allocate(self, sid, n):
        if sid in self.seqs:
            raise KeyError(sid)
        need = -(-n // self.bs)
        if need > len(self.free_ids):
            raise NoBlocks()
        self.seqs[sid] = ([self._take() for _ in range(need)], n)

    def _trim(self, sid):
        blocks, n = self.seqs[sid]
        for j in range(self._dead(n)):
            if blocks[j] is not None:
                self._drop(blocks[j])
                blocks[j] = None

    def fork(self, parent, child):
        if child in self.seqs or parent not in self.seqs:
            raise KeyError(child)
        blocks, n = self.seqs[parent]
        for b in blocks:
            if b is not None:
                self.ref[b] += 1
        self.seqs[child] = (list(blocks), n)

    def free(self, sid):
        blocks, _ = self.seqs.pop(sid)
        if sid in self.on_cpu:
            self.on_cpu.discard(sid)
            for b in reversed(blocks):
                if b is None:
                    continue
                self.cpu_ref[b] -= 1
                if self.cpu_ref[b] == 0:
                    self.cpu_free.append(b)
            return
        for b in reversed(blocks):
            if b is not None:
                self._drop(b)

    def move(self, ids, out):
        """Swap a group out (to the host pool) or in; returns the (from, to) pairs."""
        src_ref, dst_ref = (self.ref, self.cpu_ref) if out else (self.cpu_ref, self.ref)
        src_free, dst_free = (self.free_ids, self.cpu_free) if out else (self.cpu_free,
                                                                          self.free_ids)
        if len(set(ids)) != len(ids) or any((s in self.on_cpu) == out for s in ids):
            raise KeyError(ids)
        uses, order = {}, []
        for s in ids:
            for b in self.seqs[s][0]:
                if b is None:
                    continue
                if b not in uses:
                    order.append(b)
                uses[b] = uses.get(b, 0) + 1
        if any(uses[b] != src_ref[b] for b in order):
            raise KeyError("shared outside the group")
        if len(order) > len(dst_free):
            raise NoBlocks()
        moved, pairs = {}, []
        for b in order:
            nb = dst_free.pop()
            dst_ref[nb] = src_ref[b]
            src_ref[b] = 0
            src_free.append(b)
            moved[b] = nb
            pairs.append((b, nb))
        for s in ids:
            blocks, n = self.seqs[s]
            self.seqs[s] = ([None if b is None else moved[b] for b in blocks], n)
            if out:
                self.on_cpu.add(s)
            else:
                self.on_cpu.discard(s)
        return pairs

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
        for sid in ids:
            self._trim(sid)
        return slots, pairs
