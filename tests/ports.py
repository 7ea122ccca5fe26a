"""Rendezvous ports for the multi-process tests."""

def free_port() -> int:
    """A TCP port on 127.0.0.1 that the OS reports free (for a test's rendezvous)."""
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]
