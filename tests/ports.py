"""A free TCP port on 127.0.0.1 for the gloo rendezvous of a multi-process
test (the kernel picks one; fixed ports can collide with other jobs)."""
import socket


def free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]
