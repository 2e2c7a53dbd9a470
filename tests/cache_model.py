"""Host model of the streaming cache's replacement policies (LRU and LFU),
step by step as include/moe.h describes them, for checking the library's
hit / miss / eviction counts and for simulating policies on a routing trace."""


class CacheModel:
    """Slots start in order 0..n-1 (front = most recent); a forward touches
    its experts in ascending order, shared experts last, and a miss takes a
    slot not needed by the current forward (prefetch misses avoid the last
    forward's slots).  LRU takes the least recently used one.  LFU takes an
    empty slot if there is one, else keeps experts prefetched for their layer's
    next forward (until that forward has run), then prefers experts that their
    layer's previous forward did not use and among those the one with the fewest
    arrivals (forwards of its layer that used it when the layer's previous
    forward did not; all counts halve after every 64 x slots arrivals), the
    least recently used among equals."""

    AGE_EVERY = 64

    def __init__(self, n_slots, policy="lru"):
        self.n = n_slots
        self.policy = policy
        self.order = list(range(n_slots))          # front = MRU
        self.key = [None] * n_slots
        self.epoch_of = [0] * n_slots
        self.epoch = 0
        self.layer_fwds = {}
        self.use = {}           # key -> [arrivals, last forward of its layer, forward prefetched for]
        self.arrivals = 0
        self.hits = self.misses = self.prefetches = self.evictions = 0

    def _touch(self, s):
        self.order.remove(s)
        self.order.insert(0, s)

    def _victim(self):
        best, victim = None, None
        for s in reversed(self.order):
            if not (self.epoch == 0 or self.epoch_of[s] != self.epoch):
                continue
            k = self.key[s]
            if self.policy == "lru" or k is None:
                return s
            arrivals, last, pf = self.use.get(k, (0, 0, 0))
            lf = self.layer_fwds.get(k[0], 0)
            recent = last != 0 and lf - last < 2
            score = (pf > lf, recent, arrivals)
            if best is None or score < best:
                best, victim = score, s
        return victim

    def _fetch(self, key, pin, prefetch):
        if not prefetch and self.policy == "lfu":
            f = self.layer_fwds[key[0]]
            u = self.use.setdefault(key, [0, 0, 0])
            if u[1] == 0 or f - u[1] > 1:
                u[0] += 1
                self.arrivals += 1
                if self.arrivals % (self.AGE_EVERY * self.n) == 0:
                    for v in self.use.values():
                        v[0] >>= 1
            u[1] = f
        if prefetch and self.policy == "lfu":
            self.use.setdefault(key, [0, 0, 0])[2] = self.layer_fwds.get(key[0], 0) + 1
        if key in self.key:
            s = self.key.index(key)
            if not prefetch:
                self.hits += 1
        else:
            s = self._victim()
            if self.key[s] is not None:
                self.evictions += 1
            self.key[s] = key
            if prefetch:
                self.prefetches += 1
            else:
                self.misses += 1
        self._touch(s)
        if pin:
            self.epoch_of[s] = self.epoch

    def forward(self, layer, experts):
        self.epoch += 1
        self.layer_fwds[layer] = self.layer_fwds.get(layer, 0) + 1
        for e in sorted(set(experts)):
            self._fetch((layer, e), True, False)

    def prefetch(self, layer, experts):
        for e in experts:
            self._fetch((layer, e), False, True)
